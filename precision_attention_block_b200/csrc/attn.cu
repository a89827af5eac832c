// Fused selective mixed-precision attention forward for sm_100a (ThriftAttention technical
// summary, "Gemengd-Precisie Berekening & Samenvoeging" and the paragraph on its fused kernel).
//
// One persistent CTA per SM walks (batch, query head, 128-row query tile) units, heaviest causal
// tiles first.  For each unit the key blocks form a list of entries: first every key block that
// some row of the tile computes in NVFP4, then every key block it computes in FP16 (the order the
// pages' kernel uses; the FP16 query tile is fetched only when the first FP16 entry comes up).
// Warp roles:
//   warp 0      TMA producer: builds the unit's entry list, loads the NVFP4 query tile, the FP16
//               query tile on demand, and for every entry its K and V tiles into a page ring (one
//               page holds an NVFP4 entry's K and V, an FP16 entry takes two pages).
//   warp 1      QK^T issuer: S = Q K^T of each entry into one of two TMEM score buffers;
//               tcgen05.mma.kind::mxf4nvf4.block_scale.block16 for NVFP4 pairs (E4M3 scale
//               vectors copied into TMEM by tcgen05.cp), kind::f16 for FP16 pairs.
//   warp 2      PV issuer: the entry's probability block times V into a TMEM PV buffer.
//   warps 4-11  two softmax warpgroups; a thread of warp w owns query row 32 (w % 4) + lane of the
//               tile for one half of the keys and one half of the output columns.  Per entry both
//               read the whole score row from TMEM (so each has the row maximum M of the key block
//               without any exchange), compute P^ = exp(S - M) for their half of the keys: NVFP4
//               entries re-quantise P' = 2688 P^ with one E4M3 scale per 16 keys into shared
//               memory (the PV MMA's A operand), FP16 entries round P^ to FP16.  Then each folds
//               the previous entry's PV into its half of the row's FP32 output (registers) with
//               weight exp(M - m) and adds its half of the unquantised sum of P^ into the
//               denominator.  Part of the exponentials run as a polynomial on the FMA pipe, the
//               rest on the MUFU unit, so that neither pipe alone limits.
// Registers move from the producer warpgroup to the softmax warpgroups with setmaxnreg.
// Every wait is bounded; on timeout the CTA records THRIFT_ERR_TIMEOUT and unwinds.
#include <cuda.h>
#include <cuda_runtime.h>

#include "sm100.cuh"
#include "thrift_internal.h"

namespace thrift {

namespace {

constexpr int kBQ = 128;
constexpr long long kWaitLimit = 1ll << 32;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kSW128 = 2, kSW64 = 4, kSW32 = 6;
constexpr int kMaxPages = 8;
constexpr int kSmemLimit = 232448;  // largest dynamic shared memory of one CTA on sm_100
constexpr int kProducerRegs = 56, kSoftmaxRegs = 224;  // setmaxnreg split (384 threads x 168 at launch)
constexpr float kNegInf = -__builtin_huge_valf();
// log2 units: O and l are rescaled only when a block maximum exceeds the reference maximum by more
// than 2^32.  Until then every weight exp2(M - m_ref) is at most 2^32, so with at most 2^13 key
// blocks of at most 128 keys and |V| < 2^16 the FP32 sums stay below 2^68, far from overflow, and
// FP32 keeps its relative precision at any scale.
constexpr float kRescale = 32.0f;
constexpr int kPolyPerGroup = 6;  // exponentials per 16 keys evaluated by the polynomial (measured best)

__host__ __device__ constexpr int round1024(int x) { return (x + 1023) & ~1023; }
__host__ __device__ constexpr int swz_for_row_bytes(int b) { return b == 128 ? kSW128 : (b == 64 ? kSW64 : kSW32); }
__host__ __device__ constexpr int cmax(int a, int b) { return a > b ? a : b; }

template <int D, int BK>
struct Layout {
  // TMEM columns: PV result buffers, two score buffers, scale vectors of Q, K (x2), V (x2), P (x2)
  static constexpr int SFQ = 4 * (D / 64);
  static constexpr int SFV = 4 * (BK / 64);
  static constexpr int SF_COLS = 3 * SFQ + 4 * SFV;
  static constexpr int NPV = 2 * D + 2 * BK + SF_COLS <= 512 ? 2 : 1;  // PV buffers
  static constexpr int COL_PV = 0;
  static constexpr int COL_S = NPV * D;
  static constexpr int COL_SFQ = COL_S + 2 * BK;
  static constexpr int COL_SFK = COL_SFQ + SFQ;
  static constexpr int COL_SFV = COL_SFK + 2 * SFQ;
  static constexpr int COL_SFP = COL_SFV + 2 * SFV;
  static constexpr int TMEM_COLS = COL_SFP + 2 * SFV;
  static_assert(TMEM_COLS <= 512, "TMEM budget");
  static constexpr int THREADS = 384;
  static constexpr int KH = BK / 2;  // keys of a row per softmax warpgroup
  static constexpr int DH = D / 2;   // output columns of a row per softmax warpgroup

  // shared memory: NVFP4 query tile + its scales, FP16 query tile, two PV operand buffers
  static constexpr int Q4_BYTES = kBQ * D / 2;
  static constexpr int QSF_BYTES = (D / 64) * 512;
  static constexpr int Q4_REGION = round1024(Q4_BYTES + QSF_BYTES);
  static constexpr int Q16_BYTES = kBQ * D * 2;
  static constexpr int P4_BYTES = kBQ * BK / 2;
  static constexpr int PSF_BYTES = (BK / 64) * 512;
  static constexpr int P16_BYTES = kBQ * BK * 2;
  static constexpr int PBUF = round1024(cmax(P16_BYTES, P4_BYTES + PSF_BYTES));
  // one page: an NVFP4 entry (K codes, K scales, V codes, V scales) or one FP16 K or V tile
  static constexpr int K16_BYTES = BK * D * 2;
  static constexpr int K4_BYTES = BK * D / 2;
  static constexpr int KSF_BYTES = (D / 64) * 512;  // the 128-row scale block(s) holding the tile's rows
  static constexpr int V4_OFF = round1024(K4_BYTES + KSF_BYTES);
  static constexpr int V4_BYTES = D * BK / 2;
  static constexpr int VSF_BYTES = (BK / 64) * 512;
  static constexpr int FP4_ENTRY = V4_OFF + V4_BYTES + VSF_BYTES;
  static constexpr int PAGE = round1024(cmax(K16_BYTES, FP4_ENTRY));

  static constexpr int OFF_Q4 = 0;
  static constexpr int OFF_Q16 = OFF_Q4 + Q4_REGION;
  static constexpr int OFF_P = OFF_Q16 + Q16_BYTES;
  static constexpr int OFF_PAGES = OFF_P + 2 * PBUF;
  static constexpr int BAR_BYTES = 3072;
  // + npage pages, then the barrier block, then the entry lists (sizes chosen at launch)
  static constexpr int fixed_bytes() { return OFF_PAGES + BAR_BYTES + 1024 /* alignment slack */; }
};

struct Bars {
  uint64_t q4_full, q4_empty, q16_full, q16_empty;
  uint64_t ready[2];  // visit v: S(v) = Q K^T and the PV product of visit v - LAG are in TMEM (one
                      // commit from each issuer)
  uint64_t s_free[2], p_full[2];  // score buffer read, PV operand written (both softmax warpgroups)
  uint64_t list_full[2], list_empty[2];  // by unit parity
  uint64_t lx_bar[2];                    // the two softmax warpgroups swap their denominators
  uint64_t page_full[kMaxPages], page_empty[kMaxPages];
  int list_count[2];
  uint32_t tmem_base;
  int abort_flag;
  float lx[2][2][128];  // [unit parity][warpgroup][row] partial denominators
};
static_assert(sizeof(Bars) <= 3072, "barrier block");

struct AttnParams {
  const uint32_t* mask;
  const uint8_t* q_sf;
  const uint8_t* k_sf;
  const uint8_t* v_sf;
  const float* q_ts;
  const float* k_ts;
  const float* v_ts;
  __half* out;
  long long osb, osh, osn;  // output strides in elements ([B, Hq, N, d] view, d contiguous)
  float* out_hp;  // optional FP32 copy of the output before its FP16 rounding (Attn-QAT's O')
  float* lse;
  int* status;
  float* dbg;  // optional dump of one entry (S, P bytes, PV) of tile 0 of the first unit of CTA 0
  int dbg_entry;
  int B, Hq, Hkv, N, bq, causal, mode, nqb, nkb, mask_words, n_units;  // mode as attn_launch
  int running_max;  // first level of the P requantisation: 0 = the block maximum, 1 = the running maximum
  int npage, maxe, off_bar, off_list;
  float tau;
  long long wait_limit;
};

struct UnitInfo {
  int b, h, hk, t;
};

// The unit a CTA takes in its round r: units are ordered heaviest first (longest causal rows), and
// the CTAs take them in a snake order (CTA c takes unit r * G + c in even rounds and
// r * G + G - 1 - c in odd ones), which evens out the work per CTA.
__device__ __forceinline__ int unit_of(int r) {
  return r * (int)gridDim.x + ((r & 1) ? (int)gridDim.x - 1 - (int)blockIdx.x : (int)blockIdx.x);
}

__device__ __forceinline__ UnitInfo decode_unit(const AttnParams& p, int u) {
  const int bh_count = p.B * p.Hq;
  UnitInfo ui;
  ui.t = p.N / kBQ - 1 - u / bh_count;  // heaviest (longest causal rows) first
  const int bh = u % bh_count;
  ui.b = bh / p.Hq;
  ui.h = bh % p.Hq;
  ui.hk = ui.h / (p.Hq / p.Hkv);
  return ui;
}

// The entry list of one 128-row tile of query head h, built by a whole warp: NVFP4 entries, then
// FP16 entries, each as j | fp16 << 13 | row-half mask << 14 (with 64-row query blocks a key
// block can be NVFP4 for one half of the tile and FP16 for the other).  Returns the number of
// entries (same in every lane), at least min_entries.
template <int BK>
__device__ int build_list(const AttnParams& p, int b, int h, int t, uint16_t* list, int lane, int min_entries) {
  const bool two = p.bq == 64;
  const int i0 = two ? 2 * t : t, i1 = i0 + 1;
  const uint32_t* base = p.mask ? p.mask + ((int64_t)(b * p.Hq + h) * p.nqb) * p.mask_words : nullptr;
  const uint32_t* m0 = base ? base + (int64_t)i0 * p.mask_words : nullptr;
  const uint32_t* m1 = (base && two) ? base + (int64_t)i1 * p.mask_words : nullptr;
  int jmax0, jmax1;
  if (p.causal) {
    jmax0 = ((i0 + 1) * p.bq - 1) / BK + 1;
    jmax1 = two ? ((i1 + 1) * p.bq - 1) / BK + 1 : 0;
  } else {
    jmax0 = p.nkb;
    jmax1 = two ? p.nkb : 0;
  }
  const int jmax = jmax0 > jmax1 ? jmax0 : jmax1;
  auto sel = [&](const uint32_t* m, int jj) -> int {
    if (p.mode == 2) return 1;
    if (p.mode == 1) return 0;
    return (int)((__ldg(m + (jj >> 5)) >> (jj & 31)) & 1u);
  };
  int n = 0;
  // the sparse variant (mode 3) keeps only the FP16 (selected) entries
  for (int phase = p.mode == 3 ? 1 : 0; phase < 2; ++phase) {
    for (int jb = 0; jb < jmax; jb += 32) {
      const int jj = jb + lane;
      int rm = 0;
      if (jj < jmax0 && sel(m0, jj) == phase) rm |= 1;
      if (two && jj < jmax1 && sel(m1, jj) == phase) rm |= 2;
      if (!two && rm) rm = 3;
      const unsigned bal = __ballot_sync(0xffffffffu, rm != 0);
      if (rm && THRIFT_CHECK(n + __popc(bal) <= p.maxe, p.status))
        list[n + __popc(bal & ((1u << lane) - 1u))] = (uint16_t)(jj | (phase << 13) | (rm << 14));
      n += __popc(bal);
    }
  }
  // The softmax warpgroups merge a tile's last PV products (the last min_entries visits, which lag
  // that far behind S) while they wait for the next tile's first min_entries visits; those must
  // come from the next list, since the list after it is built only once this tile is released.
  // A shorter list (the sparse variant's empty tiles; a first causal tile with a single key block)
  // is padded with entries in which no row takes part (rm = 0: every probability is 0), NVFP4
  // ones when only NVFP4 operands exist, FP16 ones otherwise.
  if (n < min_entries) {
    if (lane < min_entries - n) list[n + lane] = (uint16_t)(p.mode == 1 ? 0 : (1 << 13));
    __syncwarp();
    n = min_entries;
  }
  return n;
}

// Page ring position shared by the producer and both issuers (same sequence of pages).
struct PageRing {
  int idx, phase, n;
  __device__ __forceinline__ void next(int& i, int& ph) {
    i = idx;
    ph = phase;
    if (++idx == n) {
      idx = 0;
      phase ^= 1;
    }
  }
};

__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProducerRegs));
}
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA pipe: x = n + f with n = round(x) (by the 1.5 * 2^23 rounding constant) and f in
// [-1/2, 1/2]; 2^f by a degree-5 polynomial whose coefficients are a relative-error minimax fit
// on [-1/2, 1/2] (Lawson's iteratively reweighted least squares over Chebyshev-spaced nodes,
// rounded to FP32; relative error below 2.2e-7 including FP32 rounding, about that of the MUFU
// ex2 approximation, so the E2M1 code decisions of the two paths agree as often); n is added to
// the exponent field.  Inputs are clamped at -125 so that the result stays a normal number
// (2^-125 is far below anything that can change a sum or a code).
__device__ __forceinline__ float ex2_poly1(float x) {
  x = fmaxf(x, -125.0f);
  const float t = x + 12582912.0f;
  const float n = t - 12582912.0f;
  const float f = x - n;
  float q = fmaf(0.0013276473619043827f, f, 0.009675541892647743f);
  q = fmaf(q, f, 0.05550713092088699f);
  q = fmaf(q, f, 0.24022120237350464f);
  q = fmaf(q, f, 0.6931469440460205f);
  q = fmaf(q, f, 1.0000001192092896f);
  return __int_as_float(__float_as_int(q) + (__float_as_int(t) << 23));
}

__device__ __forceinline__ float2 ex2_pair(float2 x, int pair) {
  if (2 * pair >= 16 - kPolyPerGroup) return make_float2(ex2_poly1(x.x), ex2_poly1(x.y));
  return make_float2(ex2(x.x), ex2(x.y));
}

__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
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

// Two non-negative FP32 values to E4M3 (round to nearest even, saturating): lo in bits 0-7, hi in 8-15.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t out;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(hi), "f"(lo));
  return out;
}

// Two E4M3 codes (bits 0-7, 8-15) back to FP32, exactly (through FP16).
__device__ __forceinline__ float2 e4m3x2_to_f32(uint32_t c2) {
  uint32_t h2;
  asm("{\n\t.reg .b16 c;\n\tcvt.u16.u32 c, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, c;\n\t}" : "=r"(h2) : "r"(c2));
  __half2 h = *reinterpret_cast<__half2*>(&h2);
  return __half22float2(h);
}

// Keys above the query become -inf (causal, on a diagonal block).
template <int n>
__device__ __forceinline__ void mask_causal(float (&s)[n], int key0, int row) {
#pragma unroll
  for (int i = 0; i < n; ++i) s[i] = (key0 + i > row) ? kNegInf : s[i];
}

template <int n>
__device__ __forceinline__ void group_max(const float (&s)[n], float* gm) {
#pragma unroll
  for (int q = 0; q < n / 16; ++q) {
    const float* x = s + 16 * q;
    const float a = max3(x[0], x[1], x[2]), b = max3(x[3], x[4], x[5]), c = max3(x[6], x[7], x[8]);
    const float d = max3(x[9], x[10], x[11]), e = max3(x[12], x[13], x[14]);
    gm[q] = max3(max3(a, b, c), max3(d, e, x[15]), kNegInf);
  }
}

// NVFP4 re-quantisation of 32 keys (two 16-key groups) of one row:
//   P^ = exp2(s*sl2 - Ms); per group s_b = E4M3(2688 max(P^) / 6); codes = E2M1(2688 P^ / s_b).
// log2(2688 / s_b) is folded into the exponent, so each key costs one FMA and one exp2.  A group
// whose scale underflows to 0 gets all-zero codes (its values are below 2688 * 2^-10 / 6 / 448).
// Returns the FP32 sum of the unquantised P^; writes 4 code words and the 2 scale bytes (sf2).
__device__ __forceinline__ float probs_nvfp4_32(const float (&s)[32], const float* gm, float sl2, float Ms,
                                                uint32_t (&cw)[4], uint32_t& sf2) {
  const float pm0 = gm[0] != kNegInf ? 448.0f * ex2(fmaf(gm[0], sl2, -Ms)) : 0.0f;
  const float pm1 = gm[1] != kNegInf ? 448.0f * ex2(fmaf(gm[1], sl2, -Ms)) : 0.0f;
  sf2 = cvt_e4m3x2(pm0, pm1);
  const float2 sbd = e4m3x2_to_f32(sf2);
  float sum = 0.0f;
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const float sbf = q ? sbd.y : sbd.x;
    const float sbe = sbf > 0.0f ? sbf : 448.0f;
    const float bias = gm[q] != kNegInf ? (11.392317422778761f - lg2(sbe)) - Ms : kNegInf;  // log2(2688/s_b) - Ms
    float y[16];
    float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
    for (int t = 0; t < 16; t += 2) {
      const float2 x = make_float2(fmaf(s[16 * q + t], sl2, bias), fmaf(s[16 * q + t + 1], sl2, bias));
      const float2 e = ex2_pair(x, t >> 1);
      y[t] = e.x;
      y[t + 1] = e.y;
      if (t & 2) { acc1.x += e.x; acc1.y += e.y; } else { acc0.x += e.x; acc0.y += e.y; }
    }
    cw[2 * q] = cvt_e2m1x8(y);
    cw[2 * q + 1] = cvt_e2m1x8(y + 8);
    sum = fmaf((acc0.x + acc1.x) + (acc0.y + acc1.y), sbe * (1.0f / 2688.0f), sum);
  }
  return sum;
}

// FP16 probabilities of 32 keys: exp2(s * sl2 - Ms) rounded to FP16 pairs, written straight into
// the SW128 PV operand row at `rowaddr` (16-byte chunk c8 at ((c8 ^ swz) << 4), chunks c0..c0+3);
// returns their FP32 sum.  `dbg` (may be null) receives the 16 words as well.
__device__ __forceinline__ float probs_fp16_32(const float (&s)[32], float sl2, float Ms, uint32_t rowaddr, int c0,
                                               int swz, uint32_t* dbg) {
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int c8 = 0; c8 < 4; ++c8) {
    uint32_t hw[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = 8 * c8 + 2 * k;
      const float2 x = make_float2(fmaf(s[i], sl2, -Ms), fmaf(s[i + 1], sl2, -Ms));
      const float2 pr = ex2_pair(x, (4 * c8 + k) & 7);
      acc[k & 1] += pr.x;
      acc[2 + (k & 1)] += pr.y;
      hw[k] = pack_half2(pr.x, pr.y);
    }
    st_shared_v4(rowaddr + (((c0 + c8) ^ swz) << 4), hw[0], hw[1], hw[2], hw[3]);
    if (dbg)
      for (int k = 0; k < 4; ++k) dbg[4 * c8 + k] = hw[k];
  }
  return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

// Maximum of n values.
template <int n>
__device__ __forceinline__ float row_max(const float* x) {
  float m = kNegInf;
#pragma unroll
  for (int i = 0; i + 2 < n; i += 3) m = max3(m, x[i], fmaxf(x[i + 1], x[i + 2]));
#pragma unroll
  for (int i = n - n % 3; i < n; ++i) m = fmaxf(m, x[i]);
  return m;
}

template <int D, int BK, bool DBG>
__global__ void __launch_bounds__(384, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm_q4, const __grid_constant__ CUtensorMap tm_k4,
                const __grid_constant__ CUtensorMap tm_v4, const __grid_constant__ CUtensorMap tm_q16,
                const __grid_constant__ CUtensorMap tm_k16, const __grid_constant__ CUtensorMap tm_v16,
                const __grid_constant__ AttnParams p) {
  using L = Layout<D, BK>;
  constexpr int KH = L::KH, DH = L::DH;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023) & ~1023u) - raw_addr);
  Bars* bars = reinterpret_cast<Bars*>(smem + p.off_bar);
  uint16_t* lists = reinterpret_cast<uint16_t*>(smem + p.off_list);  // [unit parity][maxe]
  volatile int* abort_flag = &bars->abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q4_full, 1);
    mbar_init(&bars->q4_empty, 1);
    mbar_init(&bars->q16_full, 1);
    mbar_init(&bars->q16_empty, 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars->ready[x], 2);
      mbar_init(&bars->s_free[x], 256);
      mbar_init(&bars->p_full[x], 256);
      mbar_init(&bars->list_full[x], 1);
      mbar_init(&bars->list_empty[x], 2 + 256);
      mbar_init(&bars->lx_bar[x], 256);
    }
    for (int i = 0; i < kMaxPages; ++i) {
      mbar_init(&bars->page_full[i], 1);
      mbar_init(&bars->page_empty[i], 2);
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

  if (warp < 4) {
    setmaxnreg_dec();
    if (warp == 0) {
      // ---------------------------------------------------------------- producer
      if (lane == 0) {
        if (p.mode <= 1) {
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
      PageRing ring{0, 0, p.npage};
      uint32_t uc = 0, u16c = 0;
      bool ok = true;
      for (int r = 0, u = unit_of(0); u < p.n_units && ok; u = unit_of(++r), ++uc) {
        const UnitInfo ui = decode_unit(p, u);
        const uint32_t lb = uc & 1, lph = (uc >> 1) & 1;
        // the warp is converged here: every exit below is taken by all 32 lanes together
        const bool free_ok = mbar_wait(&bars->list_empty[lb], lph ^ 1, abort_flag, p.status, lim);
        if (!__all_sync(0xffffffffu, free_ok)) break;
        uint16_t* list = lists + lb * p.maxe;
        const int n = build_list<BK>(p, ui.b, ui.h, ui.t, list, lane, L::NPV);
        __syncwarp();
        if (lane == 0) {
          bars->list_count[lb] = n;
          mbar_arrive(&bars->list_full[lb]);
          const int kvh = ui.b * p.Hkv + ui.hk;
          const int qrow0 = (ui.b * p.Hq + ui.h) * p.N + ui.t * kBQ;
          if ((ok = mbar_wait(&bars->q4_empty, (uc & 1) ^ 1, abort_flag, p.status, lim))) {
            uint8_t* sq = smem + L::OFF_Q4;
            if (p.mode <= 1) {
              mbar_arrive_expect_tx(&bars->q4_full, L::Q4_BYTES + L::QSF_BYTES);
              tma_load_2d(sq, &tm_q4, &bars->q4_full, 0, qrow0);
              bulk_load(sq + L::Q4_BYTES, p.q_sf + (size_t)(qrow0 / 128) * L::QSF_BYTES, L::QSF_BYTES, &bars->q4_full);
            } else {
              mbar_arrive(&bars->q4_full);
            }
          }
          bool q16_loaded = false;
          for (int e = 0; e < n && ok; ++e) {
            const uint32_t xe = list[e];
            const int j = xe & 0x1fff, f16 = (xe >> 13) & 1;
            const int krow0 = kvh * p.N + j * BK;
            // the tiles of this entry lie inside the tensors
            if (!THRIFT_CHECK(j < p.nkb && (ui.t + 1) * kBQ <= p.N && ui.hk < p.Hkv && ui.b < p.B, p.status)) {
              *abort_flag = 1;
              ok = false;
              break;
            }
            if (f16 && !q16_loaded) {
              if (!(ok = mbar_wait(&bars->q16_empty, (u16c & 1) ^ 1, abort_flag, p.status, lim))) break;
              ++u16c;
              uint8_t* sq = smem + L::OFF_Q16;
              mbar_arrive_expect_tx(&bars->q16_full, L::Q16_BYTES);
#pragma unroll
              for (int cb = 0; cb < D / 64; ++cb)
                tma_load_4d(sq + cb * kBQ * 128, &tm_q16, &bars->q16_full, cb * 64, ui.t * kBQ, ui.h, ui.b);
              q16_loaded = true;
            }
            int pg, ph;
            if (f16) {
              for (int kv = 0; kv < 2 && ok; ++kv) {
                ring.next(pg, ph);
                if (!(ok = mbar_wait(&bars->page_empty[pg], ph ^ 1, abort_flag, p.status, lim))) break;
                uint8_t* dst = smem + L::OFF_PAGES + pg * L::PAGE;
                mbar_arrive_expect_tx(&bars->page_full[pg], L::K16_BYTES);
#pragma unroll
                for (int cb = 0; cb < D / 64; ++cb)
                  tma_load_4d(dst + cb * BK * 128, kv ? &tm_v16 : &tm_k16, &bars->page_full[pg], cb * 64, j * BK,
                              ui.hk, ui.b);
              }
            } else {
              ring.next(pg, ph);
              if (!(ok = mbar_wait(&bars->page_empty[pg], ph ^ 1, abort_flag, p.status, lim))) break;
              uint8_t* dst = smem + L::OFF_PAGES + pg * L::PAGE;
              mbar_arrive_expect_tx(&bars->page_full[pg], L::K4_BYTES + L::KSF_BYTES + L::V4_BYTES + L::VSF_BYTES);
              tma_load_2d(dst, &tm_k4, &bars->page_full[pg], 0, krow0);
              bulk_load(dst + L::K4_BYTES, p.k_sf + (size_t)(krow0 / 128) * L::KSF_BYTES, L::KSF_BYTES,
                        &bars->page_full[pg]);
              const int vrow0 = kvh * D;
              tma_load_2d(dst + L::V4_OFF, &tm_v4, &bars->page_full[pg], j * (BK / 2), vrow0);
              const size_t sf_off = ((size_t)(vrow0 / 128) * (p.N / 64) + (size_t)j * (BK / 64)) * 512;
              bulk_load(dst + L::V4_OFF + L::V4_BYTES, p.v_sf + sf_off, L::VSF_BYTES, &bars->page_full[pg]);
            }
          }
        }
        __syncwarp();
        ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
      }
    } else if (warp == 1) {
      // ---------------------------------------------------------------- QK^T issuer
      // S = Q K^T of every visit v (a global visit counter over this CTA's units), then its commit
      // to ready[v & 1]; the PV issuer makes the other arrival.
      if (lane == 0) {
        const uint32_t idesc_qk4 = idesc_nvf4(kBQ, BK);
        const uint32_t idesc_qk16 = idesc_f16(kBQ, BK, 0, 0);
        constexpr int SWQ = swz_for_row_bytes(D / 2);
        const uint32_t qb4 = smem_u32(smem + L::OFF_Q4), qb16 = smem_u32(smem + L::OFF_Q16);
        PageRing ring{0, 0, p.npage};
        uint32_t uc = 0, u16c = 0, v = 0;
        bool ok = true;
        for (int r = 0, u = unit_of(0); u < p.n_units && ok; u = unit_of(++r), ++uc) {
          const UnitInfo ui = decode_unit(p, u);
          const int kvh = ui.b * p.Hkv + ui.hk;
          const uint32_t lb = uc & 1, lph = (uc >> 1) & 1;
          if (!(ok = mbar_wait(&bars->list_full[lb], lph, abort_flag, p.status, lim))) break;
          const int n = bars->list_count[lb];
          const uint16_t* list = lists + lb * p.maxe;
          if (!(ok = mbar_wait(&bars->q4_full, uc & 1, abort_flag, p.status, lim))) break;
          tc_fence_after();
          if (p.mode <= 1) {
#pragma unroll
            for (int kk = 0; kk < D / 64; ++kk)
              tc_copy_sf(tmem + L::COL_SFQ + 4 * kk, make_sdesc(qb4 + L::Q4_BYTES + kk * 512, 16, 128, 0));
          }
          bool released4 = false, any16 = false;
          for (int e = 0; e < n && ok; ++e, ++v) {
            const uint32_t xe = list[e];
            const int j = xe & 0x1fff, f16 = (xe >> 13) & 1;
            if (f16 && !released4) {
              tc_commit(&bars->q4_empty);  // every NVFP4 product of this unit has been issued
              released4 = true;
            }
            if (f16 && !any16) {
              if (!(ok = mbar_wait(&bars->q16_full, u16c & 1, abort_flag, p.status, lim))) break;
              ++u16c;
              any16 = true;
            }
            int pk, phk, pv, phv;
            ring.next(pk, phk);
            if (f16) ring.next(pv, phv);
            const uint32_t buf = v & 1;
            if (!(ok = mbar_wait(&bars->page_full[pk], phk, abort_flag, p.status, lim))) break;
            if (!(ok = mbar_wait(&bars->s_free[buf], ((v >> 1) & 1) ^ 1, abort_flag, p.status, lim))) break;
            tc_fence_after();
            const uint32_t kbuf = smem_u32(smem + L::OFF_PAGES + pk * L::PAGE);
            const uint32_t dS = tmem + L::COL_S + buf * BK;
            if (f16) {
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint64_t ad = make_sdesc(qb16 + (kk >> 2) * kBQ * 128 + (kk & 3) * 32, 16, 1024, kSW128);
                const uint64_t bd = make_sdesc(kbuf + (kk >> 2) * BK * 128 + (kk & 3) * 32, 16, 1024, kSW128);
                mma_f16(dS, ad, bd, idesc_qk16, kk > 0);
              }
            } else {
              const int sfk_off = ((kvh * p.N + j * BK) & 127) >> 5;
              const uint32_t sfk = tmem + L::COL_SFK + buf * L::SFQ;
#pragma unroll
              for (int kk = 0; kk < D / 64; ++kk)
                tc_copy_sf(sfk + 4 * kk, make_sdesc(kbuf + L::K4_BYTES + kk * 512, 16, 128, 0));
#pragma unroll
              for (int kk = 0; kk < D / 64; ++kk) {
                const uint64_t ad = make_sdesc(qb4 + kk * 32, 16, 8 * (D / 2), SWQ);
                const uint64_t bd = make_sdesc(kbuf + kk * 32, 16, 8 * (D / 2), SWQ);
                mma_nvf4(dS, ad, bd, idesc_qk4, tmem + L::COL_SFQ + 4 * kk, sfk + 4 * kk + sfk_off, kk > 0);
              }
            }
            tc_commit(&bars->page_empty[pk]);  // the V page of an FP16 entry is the PV issuer's
            tc_commit(&bars->ready[buf]);
          }
          if (!ok) break;
          if (!released4) tc_commit(&bars->q4_empty);
          if (any16) tc_commit(&bars->q16_empty);
          mbar_arrive(&bars->list_empty[lb]);
        }
        // the ready phases of the visits after the last one (the softmax warpgroups' last merges);
        // each arrival waits for the barrier's previous phase, so that it cannot complete that one
        for (int d = 0; d < L::NPV && ok; ++d, ++v) {
          if (!(ok = mbar_wait(&bars->ready[v & 1], ((v >> 1) & 1) ^ 1, abort_flag, p.status, lim))) break;
          mbar_arrive(&bars->ready[v & 1]);
        }
      }
    } else if (warp == 2) {
      // ---------------------------------------------------------------- PV issuer
      // For every visit v: the PV product of visit v - LAG, then its commit to ready[v & 1].  The
      // product lags LAG visits behind S so that the softmax warpgroups merge it one iteration
      // after it was issued.  LAG more iterations after the last unit issue the remaining ones.
      if (lane == 0) {
        constexpr int LAG = L::NPV;
        const uint32_t idesc_pv4 = idesc_nvf4(kBQ, D);
        const uint32_t idesc_pv16 = idesc_f16(kBQ, D, 0, 1);
        constexpr int SWP = swz_for_row_bytes(BK / 2);
        // entry parameters of the visits whose products are still to be issued, by visit parity
        int pf16[2] = {0, 0}, ppk[2] = {0, 0}, ppv[2] = {0, 0}, pphv[2] = {0, 0}, psfv[2] = {0, 0};
        PageRing ring{0, 0, p.npage};
        uint32_t uc = 0, v = 0;
        bool ok = true;
        auto issue_pv = [&](uint32_t w) -> bool {
          const uint32_t buf = w & 1;
          const int f16 = buf ? pf16[1] : pf16[0];
          const int pk = buf ? ppk[1] : ppk[0], pv = buf ? ppv[1] : ppv[0];
          const int phv = buf ? pphv[1] : pphv[0], sfv_off = buf ? psfv[1] : psfv[0];
          const uint32_t pvb = LAG == 2 ? buf : 0;
          if (!mbar_wait(&bars->p_full[buf], (w >> 1) & 1, abort_flag, p.status, lim)) return false;
          if (!mbar_wait(&bars->page_full[pv], phv, abort_flag, p.status, lim)) return false;
          tc_fence_after();
          const uint32_t pbuf = smem_u32(smem + L::OFF_P + buf * L::PBUF);
          const uint32_t vpage = smem_u32(smem + L::OFF_PAGES + pv * L::PAGE);
          const uint32_t dPV = tmem + L::COL_PV + pvb * D;
          if (f16) {
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              const uint64_t ad = make_sdesc(pbuf + (kk >> 2) * kBQ * 128 + (kk & 3) * 32, 16, 1024, kSW128);
              const uint64_t bd = make_sdesc(vpage + kk * 16 * 128, BK * 128, 1024, kSW128);
              mma_f16(dPV, ad, bd, idesc_pv16, kk > 0);
            }
            // Both arrivals of the V page come from here, after its page_full wait: an arrival
            // issued before the page holds this entry's tile could complete the phase of the
            // page's previous use.  The K page gets the QK^T commit and this arrival.
            mbar_arrive(&bars->page_empty[pk]);
            mbar_arrive(&bars->page_empty[pv]);
            tc_commit(&bars->page_empty[pv]);
          } else {
            const uint32_t vbuf = vpage + L::V4_OFF;
            const uint32_t sfv = tmem + L::COL_SFV + buf * L::SFV, sfp = tmem + L::COL_SFP + buf * L::SFV;
#pragma unroll
            for (int kb = 0; kb < BK / 64; ++kb) {
              tc_copy_sf(sfv + 4 * kb, make_sdesc(vbuf + L::V4_BYTES + kb * 512, 16, 128, 0));
              tc_copy_sf(sfp + 4 * kb, make_sdesc(pbuf + L::P4_BYTES + kb * 512, 16, 128, 0));
            }
#pragma unroll
            for (int kb = 0; kb < BK / 64; ++kb) {
              const uint64_t ad = make_sdesc(pbuf + kb * 32, 16, 8 * (BK / 2), SWP);
              const uint64_t bd = make_sdesc(vbuf + kb * 32, 16, 8 * (BK / 2), SWP);
              mma_nvf4(dPV, ad, bd, idesc_pv4, sfp + 4 * kb, sfv + 4 * kb + sfv_off, kb > 0);
            }
            tc_commit(&bars->page_empty[pv]);  // the QK^T commit was the page's other arrival
          }
          return true;
        };
        for (int r = 0, u = unit_of(0); u < p.n_units && ok; u = unit_of(++r), ++uc) {
          const UnitInfo ui = decode_unit(p, u);
          const int sfv_off = (((ui.b * p.Hkv + ui.hk) * D) & 127) >> 5;
          const uint32_t lb = uc & 1, lph = (uc >> 1) & 1;
          if (!(ok = mbar_wait(&bars->list_full[lb], lph, abort_flag, p.status, lim))) break;
          const int n = bars->list_count[lb];
          const uint16_t* list = lists + lb * p.maxe;
          for (int e = 0; e < n && ok; ++e, ++v) {
            if (v >= (uint32_t)LAG && !(ok = issue_pv(v - LAG))) break;
            tc_commit(&bars->ready[v & 1]);
            const int f16 = (list[e] >> 13) & 1;
            int pk, phk, pv, phv;
            ring.next(pk, phk);
            pv = pk;
            phv = phk;
            if (f16) ring.next(pv, phv);
            const int k = v & 1;
            if (k) {
              pf16[1] = f16; ppk[1] = pk; ppv[1] = pv; pphv[1] = phv; psfv[1] = sfv_off;
            } else {
              pf16[0] = f16; ppk[0] = pk; ppv[0] = pv; pphv[0] = phv; psfv[0] = sfv_off;
            }
          }
          if (!ok) break;
          mbar_arrive(&bars->list_empty[lb]);
        }
        // the last LAG PV products (and the ready phases the softmax warpgroups wait for)
        for (int d = 0; d < LAG && ok; ++d, ++v) {
          if (v >= (uint32_t)LAG && !(ok = issue_pv(v - LAG))) break;
          tc_commit(&bars->ready[v & 1]);
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax / merge
    setmaxnreg_inc();
    const int wg = (warp - 4) >> 2;  // which half of the keys and of the output columns
    const int quarter = warp & 3;
    const int rr = quarter * 32 + lane;  // row of the tile = TMEM lane
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    const float q_ts = (p.mode <= 1) ? __ldg(p.q_ts) : 1.0f;
    const float k_ts = (p.mode <= 1) ? __ldg(p.k_ts) : 1.0f;
    const float v_ts = (p.mode <= 1) ? __ldg(p.v_ts) : 1.0f;
    const float sl2_4 = q_ts * k_ts * p.tau * kLog2e;
    const float sl2_16 = p.tau * kLog2e;
    const float pv4_scale = v_ts * (1.0f / 2688.0f);
    uint32_t g = 0, uc = 0;
    bool ok = true;
    for (int r = 0, u = unit_of(0); u < p.n_units && ok; u = unit_of(++r), ++uc) {
      const UnitInfo ui = decode_unit(p, u);
      const uint32_t lb = uc & 1, lph = (uc >> 1) & 1;
      if (!(ok = mbar_wait(&bars->list_full[lb], lph, abort_flag, p.status, lim))) break;
      const int n_entries = bars->list_count[lb];
      const uint16_t* list = lists + lb * p.maxe;
      if (!THRIFT_CHECK(n_entries <= p.maxe, p.status)) {
        *abort_flag = 1;
        ok = false;
        break;
      }
      const int row = ui.t * kBQ + rr;
      const int half = (p.bq == 64) ? (rr >> 6) : 0;
      float O[DH];
#pragma unroll
      for (int c = 0; c < DH; ++c) O[c] = 0.0f;
      // running state: O and l are relative to exp2(m_ref); m_ref moves only when a block's
      // maximum exceeds it by more than 2^kRescale (the final O / l does not depend on m_ref).
      // Both warpgroups see the same block maxima, so they take the same decisions.
      float m_ref = kNegInf, l_run = 0.0f;
      // running maximum of the row over the entries visited so far (log2 units), the first level
      // of the P requantisation when p.running_max is set
      float m_run = kNegInf;
      // block maximum (log2 units; -inf: the row took no part), unquantised sum and precision of
      // the entries whose PV products are still to be merged: entry e - 1 (p1) and e - 2 (p2)
      float p1_M = kNegInf, p1_sum = 0.0f, p2_M = kNegInf, p2_sum = 0.0f;
      int p1_f16 = 0, p2_f16 = 0;
      const bool dbg_unit = DBG && p.dbg && blockIdx.x == 0 && u == (int)blockIdx.x;
      const uint32_t g0 = g;
      constexpr int LAG = L::NPV;

      // iteration e: wait for ready(v) (S of entry e and the PV product of entry e - LAG), merge
      // that PV product, then the softmax of entry e; LAG more iterations merge the last entries
      for (int e = 0; e < n_entries + LAG; ++e) {
        const uint32_t v = g0 + e, buf = v & 1;
        float cur_M = kNegInf, cur_sum = 0.0f;
        int cur_f16 = 0;
        if (!(ok = mbar_wait(&bars->ready[buf], (v >> 1) & 1, abort_flag, p.status, lim))) break;
        tc_fence_after();
        if (e >= LAG) {
          // merge entry e - LAG: its PV product into this warpgroup's output columns with weight
          // exp2(pend_M - m_ref)
          const float pM = LAG == 2 ? p2_M : p1_M;
          const float pSum = LAG == 2 ? p2_sum : p1_sum;
          const int pF16 = LAG == 2 ? p2_f16 : p1_f16;
          const uint32_t pvb = LAG == 2 ? buf : 0;
          const bool need = pM != kNegInf && (m_ref == kNegInf || pM > m_ref + kRescale);
          if (__any_sync(0xffffffffu, need)) {
            const float alpha = need ? (m_ref == kNegInf ? 0.0f : ex2(m_ref - pM)) : 1.0f;
            const float2 a2 = make_float2(alpha, alpha);
            l_run *= alpha;
#pragma unroll
            for (int c = 0; c < DH; c += 2) {
              const float2 o = __fmul2_rn(make_float2(O[c], O[c + 1]), a2);
              O[c] = o.x;
              O[c + 1] = o.y;
            }
            if (need) m_ref = pM;
          }
          const float gs = (pM == kNegInf) ? 0.0f : ex2(pM - m_ref);
          l_run = fmaf(gs, pSum, l_run);
          const float gpv = pF16 ? gs : gs * pv4_scale;
          const float2 g2 = make_float2(gpv, gpv);
          uint32_t r[DH];
#pragma unroll
          for (int c = 0; c < DH; c += 32)
            tmem_ld32(tl + L::COL_PV + pvb * D + wg * DH + c, *reinterpret_cast<uint32_t(*)[32]>(&r[c]));
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < DH; i += 2) {
            const float2 o = __ffma2_rn(g2, make_float2(__uint_as_float(r[i]), __uint_as_float(r[i + 1])),
                                        make_float2(O[i], O[i + 1]));
            O[i] = o.x;
            O[i + 1] = o.y;
          }
          if constexpr (DBG) {
            if (dbg_unit && e - LAG == p.dbg_entry)
              for (int i = 0; i < DH; ++i) p.dbg[kBQ * BK + kBQ * (BK / 2) + rr * D + wg * DH + i] = __uint_as_float(r[i]);
          }
        }
        if (e < n_entries) {
          const uint32_t xe = list[e];
          const int j = xe & 0x1fff, f16 = (xe >> 13) & 1, rm = xe >> 14;
          const bool part = (rm >> half) & 1;
          const bool diag = p.causal && (j * BK + BK - 1 > ui.t * kBQ);
          const float sl2 = f16 ? sl2_16 : sl2_4;
          const bool dumpP = dbg_unit && e == p.dbg_entry;
          const uint32_t tS = tl + L::COL_S + buf * BK;
          const int k_mine = wg * KH, k_other = KH - k_mine;
          // the other warpgroup's keys only contribute to the block maximum
          float M;
          float sm[KH];
          {
            float so[KH];
#pragma unroll
            for (int c = 0; c < KH; c += 32)
              tmem_ld32(tS + k_other + c, *reinterpret_cast<uint32_t(*)[32]>(&so[c]));
            if constexpr (BK == 128) {
              tmem_wait_ld();
              if (diag) mask_causal(so, j * BK + k_other, row);
              M = row_max<KH>(so);
            }
#pragma unroll
            for (int c = 0; c < KH; c += 32)
              tmem_ld32(tS + k_mine + c, *reinterpret_cast<uint32_t(*)[32]>(&sm[c]));
            tmem_wait_ld();
            if constexpr (BK == 64) {
              if (diag) mask_causal(so, j * BK + k_other, row);
              M = row_max<KH>(so);
            }
          }
          tc_fence_before();
          mbar_arrive(&bars->s_free[buf]);
          if constexpr (DBG) {
            if (dumpP)  // raw scores before masking; the other half comes from the other warpgroup
              for (int i = 0; i < KH; ++i) p.dbg[rr * BK + k_mine + i] = sm[i];
          }
          if (diag) mask_causal(sm, j * BK + k_mine, row);
          float gm[KH / 16];
          group_max(sm, gm);
#pragma unroll
          for (int q = 0; q < KH / 16; ++q) M = fmaxf(M, gm[q]);
          // a row outside the entry's query block (64-row query blocks) takes no part: all of its
          // group maxima become -inf, which zeroes its codes, its FP16 probabilities and its sum
          if (!part) {
            M = kNegInf;
#pragma unroll
            for (int q = 0; q < KH / 16; ++q) gm[q] = kNegInf;
          }
          const bool valid = M != kNegInf;  // false when every key of the block is masked for this row
          float Ms = valid ? M * sl2 : __builtin_huge_valf();  // +inf zeroes every probability
          if (p.running_max && valid) {
            Ms = fmaxf(Ms, m_run);
            m_run = Ms;
          }

          // this warpgroup's probabilities, 32 keys at a time, into PV operand buffer `buf`; its
          // previous reader, the PV product of entry e - 2, has completed (ready(v) covers it)
          const uint32_t pb = smem_u32(smem + L::OFF_P + buf * L::PBUF);
          float sum = 0.0f;
#pragma unroll
          for (int c = 0; c < KH; c += 32) {
            const int k0 = k_mine + c;  // first key of this chunk within the block
            const float(&sc)[32] = *reinterpret_cast<const float(*)[32]>(&sm[c]);
            if (f16) {
              uint32_t* dbw = nullptr;
              if constexpr (DBG) {
                if (dumpP) dbw = reinterpret_cast<uint32_t*>(p.dbg + kBQ * BK + rr * (BK / 2)) + k0 / 2;
              }
              sum += probs_fp16_32(sc, sl2, Ms, pb + (k0 >> 6) * kBQ * 128 + rr * 128, (k0 & 63) >> 3, rr & 7, dbw);
            } else {
              uint32_t cw[4], sf2 = 0u;
              sum += probs_nvfp4_32(sc, gm + c / 16, sl2, Ms, cw, sf2);
              const int q = k0 >> 5;  // 16-byte chunk of the row's codes
              const uint32_t addr = BK == 64 ? pb + rr * 32 + ((q ^ ((rr >> 2) & 1)) << 4)
                                             : pb + rr * 64 + ((q ^ ((rr >> 1) & 3)) << 4);
              st_shared_v4(addr, cw[0], cw[1], cw[2], cw[3]);
              const int g16 = k0 >> 4;  // first 16-key group of the chunk
              asm volatile("st.shared.b16 [%0], %1;" ::"r"(pb + L::P4_BYTES + (g16 >> 2) * 512 + (rr & 31) * 16 +
                                                            (rr >> 5) * 4 + (g16 & 3)),
                           "h"((uint16_t)sf2)
                           : "memory");
              if constexpr (DBG) {
                if (dumpP) {
                  uint8_t* db = reinterpret_cast<uint8_t*>(p.dbg + kBQ * BK + rr * (BK / 2));
                  for (int i = 0; i < 4; ++i) reinterpret_cast<uint32_t*>(db)[(k0 >> 3) + i] = cw[i];
                  db[BK / 2 + g16] = (uint8_t)sf2;
                  db[BK / 2 + g16 + 1] = (uint8_t)(sf2 >> 8);
                }
              }
            }
          }
          // the TMEM reads of this iteration's merge are complete (tcgen05.wait::ld above), so
          // this arrival also releases the PV buffer for the product of entry e
          tc_fence_before();
          fence_proxy_async_smem();
          mbar_arrive(&bars->p_full[buf]);
          cur_M = valid ? Ms : kNegInf;
          cur_sum = sum;
          cur_f16 = f16;
        }
        p2_M = p1_M;
        p2_sum = p1_sum;
        p2_f16 = p1_f16;
        p1_M = cur_M;
        p1_sum = cur_sum;
        p1_f16 = cur_f16;
      }
      if (!ok) break;
      g = g0 + n_entries;
      mbar_arrive(&bars->list_empty[lb]);
      // the two warpgroups' partial denominators (same m_ref in both), then the epilogue:
      // O / l in FP16, lse in natural-log units of the tau-scaled scores
      bars->lx[lb][wg][rr] = l_run;
      mbar_arrive(&bars->lx_bar[lb]);
      if (!(ok = mbar_wait(&bars->lx_bar[lb], lph, abort_flag, p.status, lim))) break;
      const float l_tot = bars->lx[lb][0][rr] + bars->lx[lb][1][rr];
      const float inv_l = l_tot > 0.0f ? 1.0f / l_tot : 0.0f;
      const int64_t orow = (int64_t)(ui.b * p.Hq + ui.h) * p.N + row;
      uint4* dst = reinterpret_cast<uint4*>(p.out + ui.b * p.osb + ui.h * p.osh + row * p.osn + wg * DH);
#pragma unroll
      for (int c = 0; c < DH / 8; ++c) {
        uint4 v;
        v.x = pack_half2(O[8 * c] * inv_l, O[8 * c + 1] * inv_l);
        v.y = pack_half2(O[8 * c + 2] * inv_l, O[8 * c + 3] * inv_l);
        v.z = pack_half2(O[8 * c + 4] * inv_l, O[8 * c + 5] * inv_l);
        v.w = pack_half2(O[8 * c + 6] * inv_l, O[8 * c + 7] * inv_l);
        dst[c] = v;
      }
      if (p.out_hp) {
        float4* dh = reinterpret_cast<float4*>(p.out_hp + orow * D + wg * DH);
#pragma unroll
        for (int c = 0; c < DH / 4; ++c)
          dh[c] = make_float4(O[4 * c] * inv_l, O[4 * c + 1] * inv_l, O[4 * c + 2] * inv_l, O[4 * c + 3] * inv_l);
      }
      if (p.lse && wg == 0) p.lse[orow] = (m_ref + __log2f(l_tot)) * kLn2;
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

// 4D map over an FP16 [B, H, N, D] tensor with row strides `rows` (D contiguous), boxes of 64
// channels x box_rows tokens of one (batch, head).
bool make_map4(CUtensorMap* m, const void* base, const RowMap& rows, int B, int H, int N, int D, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)N, (cuuint64_t)H, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)rows.sn * 2, (cuuint64_t)rows.sh * 2, (cuuint64_t)rows.sb * 2};
  cuuint32_t box[4] = {64, box_rows, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
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
                       const thrift_nvfp4* v4, const AttnRows& rows, AttnParams& prm, cudaStream_t stream) {
  using L = Layout<D, BK>;
  // entry lists: [unit parity][maxe] u16 after the barrier block; the rest goes to pages
  prm.maxe = (prm.bq == 64 ? 2 : 1) * prm.nkb;
  if (prm.maxe < L::NPV) prm.maxe = L::NPV;  // lists are padded to NPV entries
  const int list_bytes = (2 * prm.maxe * 2 + 1023) & ~1023;
  const int room = kSmemLimit - L::fixed_bytes() - list_bytes;
  int npage = room / L::PAGE;
  if (npage > kMaxPages) npage = kMaxPages;
  if (npage < 3) return THRIFT_ERR_UNSUPPORTED;
  prm.npage = npage;
  prm.off_bar = L::OFF_PAGES + npage * L::PAGE;
  prm.off_list = prm.off_bar + L::BAR_BYTES;
  const int smem_bytes = prm.off_list + list_bytes + 1024;
  prm.n_units = prm.B * prm.Hq * (prm.N / kBQ);

  CUtensorMap maps[6];
  memset(maps, 0, sizeof(maps));
  const uint64_t qrows = (uint64_t)prm.B * prm.Hq * prm.N, krows = (uint64_t)prm.B * prm.Hkv * prm.N;
  bool ok = true;
  if (prm.mode <= 1) {
    ok &= make_map(&maps[0], q4->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, D / 2, qrows, D / 2, kBQ, swz_enum(D / 2));
    ok &= make_map(&maps[1], k4->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, D / 2, krows, D / 2, BK, swz_enum(D / 2));
    ok &= make_map(&maps[2], v4->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)prm.N / 2,
                   (uint64_t)prm.B * prm.Hkv * D, BK / 2, D, swz_enum(BK / 2));
  }
  if (prm.mode != 1) {
    ok &= make_map4(&maps[3], q, rows.q, prm.B, prm.Hq, prm.N, D, kBQ);
    ok &= make_map4(&maps[4], k, rows.k, prm.B, prm.Hkv, prm.N, D, BK);
    ok &= make_map4(&maps[5], v, rows.v, prm.B, prm.Hkv, prm.N, D, BK);
  }
  if (!ok) return THRIFT_ERR_CUDA;
  auto kern = prm.dbg ? attn_kernel<D, BK, true> : attn_kernel<D, BK, false>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes) != cudaSuccess)
    return THRIFT_ERR_CUDA;
  {
    // setmaxnreg.inc waits until the registers it asks for are free in the CTA's launch
    // allocation; refuse to launch unless the split fits that allocation.
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return THRIFT_ERR_CUDA;
    if ((long)fa.numRegs * L::THREADS < 128L * kProducerRegs + 256L * kSoftmaxRegs) return THRIFT_ERR_UNSUPPORTED;
  }
  int grid = num_sms();
  if (grid > prm.n_units) grid = prm.n_units;
  kern<<<grid, L::THREADS, smem_bytes, stream>>>(maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], prm);
  return cudaPeekAtLastError() == cudaSuccess ? THRIFT_OK : THRIFT_ERR_CUDA;
}

// y = 2^x by the kernel's polynomial (which = 0) or the MUFU approximation (which = 1).
__global__ void ex2_probe_kernel(const float* x, float* y, int64_t n, int which) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    y[i] = which == 0 ? ex2_poly1(x[i]) : ex2(x[i]);
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
                              void* out, float* out_hp, float* lse, int running_max, const thrift_cfg& c, int* status,
                              float* dbg, int dbg_entry, cudaStream_t stream, const AttnRows* rows_in) {
  const AttnRows rows = rows_in ? *rows_in : dense_attn_rows(c);
  AttnParams prm;
  memset(&prm, 0, sizeof(prm));
  prm.mask = mask;
  if (mode <= 1) {
    prm.q_sf = q4->scales_mma;
    prm.k_sf = k4->scales_mma;
    prm.v_sf = v4->scales_mma;
    prm.q_ts = q4->tensor_scale;
    prm.k_ts = k4->tensor_scale;
    prm.v_ts = v4->tensor_scale;
  }
  prm.out = reinterpret_cast<__half*>(out);
  prm.osb = rows.out.sb;
  prm.osh = rows.out.sh;
  prm.osn = rows.out.sn;
  prm.out_hp = out_hp;
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
  prm.running_max = running_max;
  prm.nqb = c.N / c.block_q;
  prm.nkb = c.N / c.block_k;
  prm.mask_words = (prm.nkb + 31) / 32;
  prm.tau = c.softmax_scale > 0.0f ? c.softmax_scale : 1.0f / sqrtf((float)c.d);
  if (prm.nkb > 8191) return THRIFT_ERR_UNSUPPORTED;  // key-block index field of an entry
  prm.wait_limit = kWaitLimit;
  if (c.d == 128 && c.block_k == 64) return launch_t<128, 64>(q, k, v, q4, k4, v4, rows, prm, stream);
  if (c.d == 128 && c.block_k == 128) return launch_t<128, 128>(q, k, v, q4, k4, v4, rows, prm, stream);
  if (c.d == 64 && c.block_k == 64) return launch_t<64, 64>(q, k, v, q4, k4, v4, rows, prm, stream);
  if (c.d == 64 && c.block_k == 128) return launch_t<64, 128>(q, k, v, q4, k4, v4, rows, prm, stream);
  return THRIFT_ERR_UNSUPPORTED;
}

AttnRows dense_attn_rows(const thrift_cfg& c) {
  AttnRows r;
  r.q = dense_rows(c.Hq, c.N, c.d);
  r.k = dense_rows(c.Hkv, c.N, c.d);
  r.v = dense_rows(c.Hkv, c.N, c.d);
  r.out = dense_rows(c.Hq, c.N, c.d);
  return r;
}

thrift_status ex2_probe_launch(const float* x, float* y, int64_t n, int which, cudaStream_t stream) {
  int grid = num_sms() * 4;
  ex2_probe_kernel<<<grid, 256, 0, stream>>>(x, y, n, which);
  return cudaPeekAtLastError() == cudaSuccess ? THRIFT_OK : THRIFT_ERR_CUDA;
}

thrift_status wait_timeout_launch(int* status, long long limit, cudaStream_t stream) {
  wait_timeout_kernel<<<1, 32, 0, stream>>>(status, limit);
  return cudaPeekAtLastError() == cudaSuccess ? THRIFT_OK : THRIFT_ERR_CUDA;
}

}  // namespace thrift
