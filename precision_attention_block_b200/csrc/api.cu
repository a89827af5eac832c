// The C ABI of libthrift (include/thrift.h): argument checks, workspace layout, launches on the
// caller's stream.  The library allocates nothing; every buffer belongs to the caller.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "../../include/thrift.h"
#include "../../include/thrift_debug.h"
#include "thrift_internal.h"

namespace thrift {

unsigned long long current_context_id() {
  typedef CUresult (*GetCurrentFn)(CUcontext*);
  typedef CUresult (*GetIdFn)(CUcontext, unsigned long long*);
  static GetCurrentFn get_current = nullptr;
  static GetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrentFn>(ptr);
    ptr = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetIdFn>(ptr);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

int num_sms() {
  // SM count of the current device, cached per device and context: a context created after
  // cudaDeviceReset (or a green context with fewer SMs) is looked up afresh.
  static std::mutex mu;
  static int cache[64] = {0};
  static unsigned long long cache_ctx[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == 0 || cache_ctx[dev] != ctx || ctx == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
    cache_ctx[dev] = ctx;
  }
  return cache[dev];
}

namespace {

bool al16(const void* p) { return reinterpret_cast<uintptr_t>(p) % 16 == 0; }

// Strides of a [B, H, N, d] view: non-negative multiples of 8 elements (16 bytes, what the tensor
// copies need), token rows at least d apart; NULL is the dense layout.
bool strides_ok(const thrift_strides* s, int d) {
  if (!s) return true;
  if (s->b < 0 || s->h < 0 || s->n < d) return false;
  return s->b % 8 == 0 && s->h % 8 == 0 && s->n % 8 == 0;
}

RowMap rows_of(const thrift_strides* s, int H, int N, int d) {
  return s ? RowMap{s->b, s->h, s->n, H} : dense_rows(H, N, d);
}

bool cfg_ok(const thrift_cfg* c) {
  if (!c) return false;
  if (c->B <= 0 || c->Hq <= 0 || c->Hkv <= 0 || c->N <= 0) return false;
  if (c->Hq % c->Hkv != 0) return false;
  if (c->causal != 0 && c->causal != 1) return false;
  if (c->topk_abs < -1) return false;
  if (c->topk_abs == -1 && (c->topk_bp < 0 || c->topk_bp > 10000)) return false;
  if (!(c->softmax_scale >= 0.0f) || std::isinf(c->softmax_scale)) return false;
  return true;
}

thrift_status cfg_supported(const thrift_cfg* c) {
  if (!cfg_ok(c)) return THRIFT_ERR_INVALID_ARG;
  if (c->d != 64 && c->d != 128) return THRIFT_ERR_UNSUPPORTED;
  if (c->block_q != 64 && c->block_q != 128) return THRIFT_ERR_UNSUPPORTED;
  if (c->block_k != 64 && c->block_k != 128) return THRIFT_ERR_UNSUPPORTED;
  if (c->N % 128 != 0 || c->N % c->block_k != 0) return THRIFT_ERR_UNSUPPORTED;
  if (c->N / c->block_k > 32767) return THRIFT_ERR_UNSUPPORTED;
  if ((int64_t)c->B * c->Hq * c->N > (int64_t)INT32_MAX / 2) return THRIFT_ERR_UNSUPPORTED;
  return THRIFT_OK;
}

int attn_mode(const thrift_cfg* c) {
  if (c->topk_abs == 0 || (c->topk_abs < 0 && c->topk_bp == 0)) return 1;
  if (c->topk_abs < 0 && c->topk_bp == 10000) return 2;
  return 0;
}

bool ws_ok(const void* ws, size_t have, size_t need) {
  return ws && (reinterpret_cast<uintptr_t>(ws) % 256 == 0) && have >= need;
}

int* status_ptr(void* ws) { return reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + kWsStatusOff); }

bool nvfp4_ok(const thrift_nvfp4* t, int axis) {
  return t && t->codes && t->scales && t->scales_mma && t->tensor_scale && t->group_axis == axis &&
         al16(t->codes) && al16(t->scales) && al16(t->scales_mma) && reinterpret_cast<uintptr_t>(t->tensor_scale) % 4 == 0;
}

struct AutoLayout {
  size_t q4c, q4s, q4m, k4c, k4s, k4m, v4c, v4s, v4m, ts, mask, counts, lists, select, bytes;
};

AutoLayout auto_layout(const thrift_cfg& c) {
  AutoLayout L;
  size_t qn = (size_t)c.B * c.Hq * c.N * c.d, kn = (size_t)c.B * c.Hkv * c.N * c.d;
  int64_t nqb = c.N / c.block_q, nkb = c.N / c.block_k;
  size_t off = kWsHeader;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  L.q4c = take(qn / 2);
  L.q4s = take(qn / 16);
  L.q4m = take(scales_mma_bytes((int64_t)c.B * c.Hq, c.N, c.d, 0));
  L.k4c = take(kn / 2);
  L.k4s = take(kn / 16);
  L.k4m = take(scales_mma_bytes((int64_t)c.B * c.Hkv, c.N, c.d, 0));
  L.v4c = take(kn / 2);
  L.v4s = take(kn / 16);
  L.v4m = take(scales_mma_bytes((int64_t)c.B * c.Hkv, c.N, c.d, 1));
  L.ts = take(3 * sizeof(float));
  L.mask = take((size_t)c.B * c.Hq * nqb * ((nkb + 31) / 32) * 4);
  L.counts = take((size_t)c.B * c.Hq * nqb * 4);
  L.lists = take((size_t)c.B * c.Hq * nqb * nkb * 2);
  L.select = take(select_layout(c).bytes);
  L.bytes = off;
  return L;
}

bool dcfg_ok(const thrift_decode_cfg* c) {
  if (!c) return false;
  if (c->B <= 0 || c->Hq <= 0 || c->Hkv <= 0 || c->Nq <= 0 || c->Nk <= 0) return false;
  if (c->Hq % c->Hkv != 0 || c->Nq > c->Nk) return false;
  if (c->causal != 0 && c->causal != 1) return false;
  if (c->topk_abs < -1) return false;
  if (c->topk_abs == -1 && (c->topk_bp < 0 || c->topk_bp > 10000)) return false;
  if (!(c->softmax_scale >= 0.0f) || std::isinf(c->softmax_scale)) return false;
  if (c->n_valid != 0 && (c->n_valid < c->Nq || c->n_valid > c->Nk)) return false;
  return true;
}

thrift_status dcfg_supported(const thrift_decode_cfg* c) {
  if (!dcfg_ok(c)) return THRIFT_ERR_INVALID_ARG;
  if (c->d != 64 && c->d != 128) return THRIFT_ERR_UNSUPPORTED;
  if (c->block_k != 64 && c->block_k != 128) return THRIFT_ERR_UNSUPPORTED;
  if (c->Nk % 128 != 0 || c->Nk % c->block_k != 0) return THRIFT_ERR_UNSUPPORTED;
  if (c->Nk / c->block_k > 32767) return THRIFT_ERR_UNSUPPORTED;
  if ((int64_t)(c->Hq / c->Hkv) * c->Nq > 16) return THRIFT_ERR_UNSUPPORTED;
  if ((int64_t)c->B * c->Hkv * c->Nk > (int64_t)INT32_MAX / 2) return THRIFT_ERR_UNSUPPORTED;
  return THRIFT_OK;
}

int decode_mode(const thrift_decode_cfg* c) {
  if (c->topk_abs == 0 || (c->topk_abs < 0 && c->topk_bp == 0)) return 1;
  if (c->topk_abs < 0 && c->topk_bp == 10000) return 2;
  return 0;
}

struct DecodeLayout {
  size_t q4c, q4s, q4m, qts, select, mask, counts, lists, part_o, part_ml, bytes;
};

DecodeLayout decode_layout(const thrift_decode_cfg& c) {
  DecodeLayout L;
  const size_t qn = (size_t)c.B * c.Hq * c.Nq * c.d;
  const size_t heads = (size_t)c.B * c.Hq, nkb = (size_t)(c.Nk / c.block_k);
  const size_t parts = (size_t)c.B * c.Hkv * decode_split_cap((int)nkb);
  size_t off = kWsHeader;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  L.q4c = take(qn / 2);
  L.q4s = take(qn / 16);
  L.q4m = take(scales_mma_bytes((int64_t)heads, c.Nq, c.d, 0));
  L.qts = take(sizeof(float));
  L.select = take(decode_select_scratch_bytes(c));
  L.mask = take(heads * ((nkb + 31) / 32) * 4);
  L.counts = take(heads * 4);
  L.lists = take(heads * nkb * 2);
  L.part_o = take(parts * 16 * c.d * sizeof(float));
  L.part_ml = take(parts * 16 * 2 * sizeof(float));
  L.bytes = off;
  return L;
}

thrift_status decode_attn_common(const void* q, const void* k, const void* v, const thrift_nvfp4* k4,
                                 const thrift_nvfp4* v4, const uint32_t* mask, void* out, float* lse,
                                 const thrift_decode_cfg* cfg, void* ws, size_t ws_bytes, cudaStream_t s,
                                 bool sparse = false) {
  const int mode = sparse ? 3 : decode_mode(cfg);
  if (!q || !out || !al16(q)) return THRIFT_ERR_INVALID_ARG;
  if (mode != 1 && (!k || !v || !al16(k) || !al16(v))) return THRIFT_ERR_INVALID_ARG;
  if (mode <= 1) {
    if (!nvfp4_ok(k4, 0) || !nvfp4_ok(v4, 1)) return THRIFT_ERR_INVALID_ARG;
    if (!al16(k4->codes) || !al16(k4->scales) || !al16(v4->codes) || !al16(v4->scales_mma))
      return THRIFT_ERR_INVALID_ARG;
  }
  if ((mode == 0 || mode == 3) && !mask) return THRIFT_ERR_INVALID_ARG;
  const DecodeLayout L = decode_layout(*cfg);
  if (!ws_ok(ws, ws_bytes, L.bytes)) return THRIFT_ERR_WORKSPACE;
  uint8_t* w = static_cast<uint8_t*>(ws);
  thrift_nvfp4 q4 = {w + L.q4c, w + L.q4s, w + L.q4m, reinterpret_cast<float*>(w + L.qts), 0};
  const thrift_decode_cfg& c = *cfg;
  if (mode <= 1) {
    unsigned int* amax = reinterpret_cast<unsigned int*>(w + kWsAmaxOff);
    thrift_status st = quantize_launch(q, dense_rows(c.Hq, c.Nq, c.d), (int64_t)c.B * c.Hq, c.Nq, c.d, &q4, amax, s);
    if (st != THRIFT_OK) return st;
  }
  DecodeArgs a;
  a.cfg = cfg;
  a.q = q;
  a.k = k;
  a.v = v;
  a.q4 = &q4;
  a.k4 = k4;
  a.v4 = v4;
  a.mask = (mode == 0 || mode == 3) ? mask : nullptr;
  a.mode = mode;
  a.out = out;
  a.lse = lse;
  a.part_o = reinterpret_cast<float*>(w + L.part_o);
  a.part_ml = reinterpret_cast<float*>(w + L.part_ml);
  a.status = status_ptr(ws);
  return decode_attn_launch(a, s);
}

}  // namespace
}  // namespace thrift

using namespace thrift;

extern "C" {

size_t thrift_nvfp4_scales_mma_bytes(int64_t outer, int32_t N, int32_t d, int32_t group_axis) {
  if (outer <= 0 || N <= 0 || d <= 0 || (group_axis != 0 && group_axis != 1)) return 0;
  return scales_mma_bytes(outer, N, d, group_axis);
}

size_t thrift_workspace_bytes(const thrift_cfg* cfg) {
  if (cfg_supported(cfg) != THRIFT_OK) return 0;
  return kWsHeader + select_layout(*cfg).bytes;
}

size_t thrift_auto_workspace_bytes(const thrift_cfg* cfg) {
  if (cfg_supported(cfg) != THRIFT_OK) return 0;
  return auto_layout(*cfg).bytes;
}

static thrift_status quantize_common(const void* x, const thrift_strides* xs, int64_t outer, int32_t H, int32_t N,
                                     int32_t d, const thrift_nvfp4* out, void* ws, size_t ws_bytes, void* stream) {
  if (!x || outer <= 0 || N <= 0 || !out || H <= 0 || outer % H != 0) return THRIFT_ERR_INVALID_ARG;
  if (out->group_axis != 0 && out->group_axis != 1) return THRIFT_ERR_INVALID_ARG;
  if (!nvfp4_ok(out, out->group_axis)) return THRIFT_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return THRIFT_ERR_UNSUPPORTED;
  if (N % 128 != 0) return THRIFT_ERR_UNSUPPORTED;
  if ((xs || out->group_axis == 1) && outer > 65535) return THRIFT_ERR_UNSUPPORTED;  // grid rows per slice
  if (!al16(x) || !strides_ok(xs, d)) return THRIFT_ERR_INVALID_ARG;
  if (!ws_ok(ws, ws_bytes, kWsHeader)) return THRIFT_ERR_WORKSPACE;
  unsigned int* amax = reinterpret_cast<unsigned int*>(static_cast<uint8_t*>(ws) + kWsAmaxOff);
  return quantize_launch(x, rows_of(xs, H, N, d), outer, N, d, out, amax, static_cast<cudaStream_t>(stream));
}

thrift_status thrift_quantize_nvfp4(const void* x, int64_t outer, int32_t N, int32_t d, const thrift_nvfp4* out,
                                    void* ws, size_t ws_bytes, void* stream) {
  return quantize_common(x, nullptr, outer, 1, N, d, out, ws, ws_bytes, stream);
}

thrift_status thrift_quantize_nvfp4_strided(const void* x, const thrift_strides* xs, int32_t B, int32_t H, int32_t N,
                                            int32_t d, const thrift_nvfp4* out, void* ws, size_t ws_bytes,
                                            void* stream) {
  if (B <= 0 || H <= 0) return THRIFT_ERR_INVALID_ARG;
  return quantize_common(x, xs, (int64_t)B * H, H, N, d, out, ws, ws_bytes, stream);
}

thrift_status thrift_block_select_strided(const void* q, const thrift_strides* qs, const void* k,
                                          const thrift_strides* ks, const thrift_cfg* cfg, uint32_t* mask,
                                          int32_t* counts, int16_t* lists, double* scores, void* ws, size_t ws_bytes,
                                          void* stream) {
  thrift_status st = cfg_supported(cfg);
  if (st != THRIFT_OK) return st;
  if (!q || !k || !mask || !counts || !lists) return THRIFT_ERR_INVALID_ARG;
  if (!al16(q) || !al16(k) || !strides_ok(qs, cfg->d) || !strides_ok(ks, cfg->d)) return THRIFT_ERR_INVALID_ARG;
  if (!ws_ok(ws, ws_bytes, thrift_workspace_bytes(cfg))) return THRIFT_ERR_WORKSPACE;
  return select_launch(q, rows_of(qs, cfg->Hq, cfg->N, cfg->d), k, rows_of(ks, cfg->Hkv, cfg->N, cfg->d), *cfg, mask,
                       counts, lists, scores, static_cast<uint8_t*>(ws) + kWsHeader, static_cast<cudaStream_t>(stream));
}

thrift_status thrift_block_select(const void* q, const void* k, const thrift_cfg* cfg, uint32_t* mask,
                                  int32_t* counts, int16_t* lists, double* scores, void* ws, size_t ws_bytes,
                                  void* stream) {
  return thrift_block_select_strided(q, nullptr, k, nullptr, cfg, mask, counts, lists, scores, ws, ws_bytes, stream);
}

thrift_status thrift_block_select_noalloc(const void* q, const void* k, const thrift_cfg* cfg, uint32_t* mask,
                                          int32_t* counts, int16_t* lists, double* scores, void* stream) {
  thrift_status st = cfg_supported(cfg);
  if (st != THRIFT_OK) return st;
  if (!q || !k || !mask || !counts || !lists) return THRIFT_ERR_INVALID_ARG;
  if (!al16(q) || !al16(k)) return THRIFT_ERR_INVALID_ARG;
  if (select_layout(*cfg).bytes > noalloc_select_scratch_bytes()) return THRIFT_ERR_WORKSPACE;
  uint8_t* scratch = nullptr;
  if ((st = noalloc_select_scratch(&scratch)) != THRIFT_OK) return st;
  const thrift_cfg& c = *cfg;
  return select_launch(q, dense_rows(c.Hq, c.N, c.d), k, dense_rows(c.Hkv, c.N, c.d), c, mask, counts, lists, scores,
                       scratch, static_cast<cudaStream_t>(stream));
}

static thrift_status attn_common(const void* q, const void* k, const void* v, const thrift_nvfp4* q4,
                                 const thrift_nvfp4* k4, const thrift_nvfp4* v4, const uint32_t* mask, void* out,
                                 float* out_hp, float* lse, int running_max, const thrift_cfg* cfg, void* ws,
                                 size_t ws_bytes, float* dbg, int dbg_entry, void* stream,
                                 const thrift_strides* qs = nullptr, const thrift_strides* ks = nullptr,
                                 const thrift_strides* vs = nullptr, const thrift_strides* os = nullptr) {
  thrift_status st = cfg_supported(cfg);
  if (st != THRIFT_OK) return st;
  const int d = cfg->d;
  if (!strides_ok(qs, d) || !strides_ok(ks, d) || !strides_ok(vs, d) || !strides_ok(os, d))
    return THRIFT_ERR_INVALID_ARG;
  AttnRows rows;
  rows.q = rows_of(qs, cfg->Hq, cfg->N, d);
  rows.k = rows_of(ks, cfg->Hkv, cfg->N, d);
  rows.v = rows_of(vs, cfg->Hkv, cfg->N, d);
  rows.out = rows_of(os, cfg->Hq, cfg->N, d);
  if (!out) return THRIFT_ERR_INVALID_ARG;
  int mode = attn_mode(cfg);
  if (mode != 2 && (!nvfp4_ok(q4, 0) || !nvfp4_ok(k4, 0) || !nvfp4_ok(v4, 1))) return THRIFT_ERR_INVALID_ARG;
  if (mode != 1 && (!q || !k || !v)) return THRIFT_ERR_INVALID_ARG;
  if (mode != 1 && (!al16(q) || !al16(k) || !al16(v))) return THRIFT_ERR_INVALID_ARG;
  if (!al16(out) || (out_hp && !al16(out_hp))) return THRIFT_ERR_INVALID_ARG;
  if (mode == 0 && !mask) return THRIFT_ERR_INVALID_ARG;
  if (!ws_ok(ws, ws_bytes, kWsHeader)) return THRIFT_ERR_WORKSPACE;
  return attn_launch_dbg(q, k, v, q4, k4, v4, mask, mode, out, out_hp, lse, running_max, *cfg, status_ptr(ws), dbg,
                         dbg_entry, static_cast<cudaStream_t>(stream), &rows);
}

thrift_status thrift_attn_fwd(const void* q, const void* k, const void* v, const thrift_nvfp4* q4,
                              const thrift_nvfp4* k4, const thrift_nvfp4* v4, const uint32_t* mask,
                              const int32_t* counts, const int16_t* lists, void* out, float* lse,
                              const thrift_cfg* cfg, void* ws, size_t ws_bytes, void* stream) {
  (void)counts;
  (void)lists;
  return attn_common(q, k, v, q4, k4, v4, mask, out, nullptr, lse, 0, cfg, ws, ws_bytes, nullptr, -1, stream);
}

thrift_status thrift_attn_fwd_strided(const void* q, const thrift_strides* qs, const void* k, const thrift_strides* ks,
                                      const void* v, const thrift_strides* vs, const thrift_nvfp4* q4,
                                      const thrift_nvfp4* k4, const thrift_nvfp4* v4, const uint32_t* mask, void* out,
                                      const thrift_strides* os, float* lse, const thrift_cfg* cfg, void* ws,
                                      size_t ws_bytes, void* stream) {
  return attn_common(q, k, v, q4, k4, v4, mask, out, nullptr, lse, 0, cfg, ws, ws_bytes, nullptr, -1, stream, qs, ks,
                     vs, os);
}

thrift_status thrift_attn_fwd_running_max(const void* q, const void* k, const void* v, const thrift_nvfp4* q4,
                                          const thrift_nvfp4* k4, const thrift_nvfp4* v4, const uint32_t* mask,
                                          void* out, float* lse, const thrift_cfg* cfg, void* ws, size_t ws_bytes,
                                          void* stream) {
  return attn_common(q, k, v, q4, k4, v4, mask, out, nullptr, lse, 1, cfg, ws, ws_bytes, nullptr, -1, stream);
}

thrift_status thrift_attn_fwd_qat(const void* q, const void* k, const void* v, const thrift_nvfp4* q4,
                                  const thrift_nvfp4* k4, const thrift_nvfp4* v4, const uint32_t* mask, void* out,
                                  float* out_hp, float* lse, const thrift_cfg* cfg, void* ws, size_t ws_bytes,
                                  void* stream) {
  if (!out_hp) return THRIFT_ERR_INVALID_ARG;
  return attn_common(q, k, v, q4, k4, v4, mask, out, out_hp, lse, 0, cfg, ws, ws_bytes, nullptr, -1, stream);
}

thrift_status thrift_debug_attn_dump(const void* q, const void* k, const void* v, const thrift_nvfp4* q4,
                                     const thrift_nvfp4* k4, const thrift_nvfp4* v4, const uint32_t* mask,
                                     void* out, float* lse, const thrift_cfg* cfg, void* ws, size_t ws_bytes,
                                     float* dbg, int32_t dbg_entry, void* stream) {
  if (!dbg) return THRIFT_ERR_INVALID_ARG;
  return attn_common(q, k, v, q4, k4, v4, mask, out, nullptr, lse, 0, cfg, ws, ws_bytes, dbg, dbg_entry, stream);
}

thrift_status thrift_attn_fwd_auto(const void* q, const void* k, const void* v, void* out, float* lse,
                                   const thrift_cfg* cfg, void* ws, size_t ws_bytes, void* stream) {
  return thrift_attn_fwd_auto_strided(q, nullptr, k, nullptr, v, nullptr, out, nullptr, lse, cfg, ws, ws_bytes,
                                      stream);
}

thrift_status thrift_attn_fwd_auto_strided(const void* q, const thrift_strides* qs, const void* k,
                                           const thrift_strides* ks, const void* v, const thrift_strides* vs,
                                           void* out, const thrift_strides* os, float* lse, const thrift_cfg* cfg,
                                           void* ws, size_t ws_bytes, void* stream) {
  thrift_status st = cfg_supported(cfg);
  if (st != THRIFT_OK) return st;
  if (!q || !k || !v || !out) return THRIFT_ERR_INVALID_ARG;
  if (!al16(q) || !al16(k) || !al16(v) || !al16(out)) return THRIFT_ERR_INVALID_ARG;
  if (!strides_ok(qs, cfg->d) || !strides_ok(ks, cfg->d) || !strides_ok(vs, cfg->d) || !strides_ok(os, cfg->d))
    return THRIFT_ERR_INVALID_ARG;
  AutoLayout L = auto_layout(*cfg);
  if (!ws_ok(ws, ws_bytes, L.bytes)) return THRIFT_ERR_WORKSPACE;
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* ts = reinterpret_cast<float*>(w + L.ts);
  thrift_nvfp4 q4 = {w + L.q4c, w + L.q4s, w + L.q4m, ts + 0, 0};
  thrift_nvfp4 k4 = {w + L.k4c, w + L.k4s, w + L.k4m, ts + 1, 0};
  thrift_nvfp4 v4 = {w + L.v4c, w + L.v4s, w + L.v4m, ts + 2, 1};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned int* amax = reinterpret_cast<unsigned int*>(w + kWsAmaxOff);
  int mode = attn_mode(cfg);
  const thrift_cfg& c = *cfg;
  AttnRows rows;
  rows.q = rows_of(qs, c.Hq, c.N, c.d);
  rows.k = rows_of(ks, c.Hkv, c.N, c.d);
  rows.v = rows_of(vs, c.Hkv, c.N, c.d);
  rows.out = rows_of(os, c.Hq, c.N, c.d);
  if (mode != 2) {
    if ((st = quantize_launch(q, rows.q, (int64_t)c.B * c.Hq, c.N, c.d, &q4, amax, s)) != THRIFT_OK) return st;
    if ((st = quantize_launch(k, rows.k, (int64_t)c.B * c.Hkv, c.N, c.d, &k4, amax, s)) != THRIFT_OK) return st;
    if ((st = quantize_launch(v, rows.v, (int64_t)c.B * c.Hkv, c.N, c.d, &v4, amax, s)) != THRIFT_OK) return st;
  }
  uint32_t* mask = reinterpret_cast<uint32_t*>(w + L.mask);
  if (mode == 0) {
    st = select_launch(q, rows.q, k, rows.k, c, mask, reinterpret_cast<int32_t*>(w + L.counts),
                       reinterpret_cast<int16_t*>(w + L.lists), nullptr, w + L.select, s);
    if (st != THRIFT_OK) return st;
  }
  return attn_launch_dbg(q, k, v, &q4, &k4, &v4, mode == 0 ? mask : nullptr, mode, out, nullptr, lse, 0, c,
                         status_ptr(ws), nullptr, -1, s, &rows);
}

thrift_status thrift_kv_block_means(const void* k, int64_t outer, int32_t Nk, int32_t d, int32_t block_k,
                                    double* kbar, void* stream) {
  if (!k || !kbar || outer <= 0 || Nk <= 0 || !al16(k)) return THRIFT_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return THRIFT_ERR_UNSUPPORTED;
  if (block_k != 64 && block_k != 128) return THRIFT_ERR_UNSUPPORTED;
  if (Nk % block_k != 0 || outer > 65535) return THRIFT_ERR_UNSUPPORTED;
  return kv_means_launch(k, outer, Nk, d, block_k, kbar, static_cast<cudaStream_t>(stream));
}

size_t thrift_decode_workspace_bytes(const thrift_decode_cfg* cfg) {
  if (dcfg_supported(cfg) != THRIFT_OK) return 0;
  return decode_layout(*cfg).bytes;
}

thrift_status thrift_decode_select(const void* q, const double* kbar, const thrift_decode_cfg* cfg, uint32_t* mask,
                                   int32_t* counts, int16_t* lists, double* scores, void* ws, size_t ws_bytes,
                                   void* stream) {
  thrift_status st = dcfg_supported(cfg);
  if (st != THRIFT_OK) return st;
  if (!q || !kbar || !mask || !counts || !lists) return THRIFT_ERR_INVALID_ARG;
  const DecodeLayout L = decode_layout(*cfg);
  if (!ws_ok(ws, ws_bytes, L.bytes)) return THRIFT_ERR_WORKSPACE;
  return decode_select_launch(q, kbar, *cfg, mask, counts, lists, scores, static_cast<uint8_t*>(ws) + L.select,
                              static_cast<cudaStream_t>(stream));
}

thrift_status thrift_decode_attn(const void* q, const void* k, const void* v, const thrift_nvfp4* k4,
                                 const thrift_nvfp4* v4, const uint32_t* mask, void* out, float* lse,
                                 const thrift_decode_cfg* cfg, void* ws, size_t ws_bytes, void* stream) {
  thrift_status st = dcfg_supported(cfg);
  if (st != THRIFT_OK) return st;
  return decode_attn_common(q, k, v, k4, v4, mask, out, lse, cfg, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

thrift_status thrift_decode_attn_sparse(const void* q, const void* k, const void* v, const uint32_t* mask, void* out,
                                        float* lse, const thrift_decode_cfg* cfg, void* ws, size_t ws_bytes,
                                        void* stream) {
  thrift_status st = dcfg_supported(cfg);
  if (st != THRIFT_OK) return st;
  return decode_attn_common(q, k, v, nullptr, nullptr, mask, out, lse, cfg, ws, ws_bytes,
                            static_cast<cudaStream_t>(stream), true);
}

thrift_status thrift_attn_fwd_sparse(const void* q, const void* k, const void* v, const uint32_t* mask,
                                     const int32_t* counts, const int16_t* lists, void* out, float* lse,
                                     const thrift_cfg* cfg, void* ws, size_t ws_bytes, void* stream) {
  (void)counts;
  (void)lists;
  thrift_status st = cfg_supported(cfg);
  if (st != THRIFT_OK) return st;
  if (!q || !k || !v || !mask || !out) return THRIFT_ERR_INVALID_ARG;
  if (!ws_ok(ws, ws_bytes, kWsHeader)) return THRIFT_ERR_WORKSPACE;
  return attn_launch_dbg(q, k, v, nullptr, nullptr, nullptr, mask, 3, out, nullptr, lse, 0, *cfg, status_ptr(ws), nullptr, -1,
                         static_cast<cudaStream_t>(stream));
}

thrift_status thrift_decode_fwd(const void* q, const void* k, const void* v, const thrift_nvfp4* k4,
                                const thrift_nvfp4* v4, const double* kbar, void* out, float* lse,
                                const thrift_decode_cfg* cfg, void* ws, size_t ws_bytes, void* stream) {
  thrift_status st = dcfg_supported(cfg);
  if (st != THRIFT_OK) return st;
  const DecodeLayout L = decode_layout(*cfg);
  if (!ws_ok(ws, ws_bytes, L.bytes)) return THRIFT_ERR_WORKSPACE;
  uint8_t* w = static_cast<uint8_t*>(ws);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* mask = reinterpret_cast<uint32_t*>(w + L.mask);
  if (decode_mode(cfg) == 0) {
    if (!q || !kbar) return THRIFT_ERR_INVALID_ARG;
    // the attention reads only the mask: no counts and lists here
    st = decode_select_launch(q, kbar, *cfg, mask, nullptr, nullptr, nullptr, w + L.select, s);
    if (st != THRIFT_OK) return st;
  }
  return decode_attn_common(q, k, v, k4, v4, mask, out, lse, cfg, ws, ws_bytes, s);
}

thrift_status thrift_nvfp4_tensor_scale(const void* x, int64_t n, float* tensor_scale, void* ws, size_t ws_bytes,
                                        void* stream) {
  if (!x || !tensor_scale || n <= 0 || n % 8 != 0 || reinterpret_cast<uintptr_t>(x) % 16 != 0)
    return THRIFT_ERR_INVALID_ARG;
  if (!ws_ok(ws, ws_bytes, kWsHeader)) return THRIFT_ERR_WORKSPACE;
  return tensor_scale_launch(x, n, tensor_scale,
                             reinterpret_cast<unsigned int*>(static_cast<uint8_t*>(ws) + kWsAmaxOff),
                             static_cast<cudaStream_t>(stream));
}

thrift_status thrift_kv_append(const void* k_new, const void* v_new, int64_t outer, int32_t Ncap, int32_t d,
                               int32_t block_k, int32_t len, int32_t T, void* k, void* v, const thrift_nvfp4* k4,
                               const thrift_nvfp4* v4, double* kbar, void* stream) {
  if (!k || !v || !kbar || !nvfp4_ok(k4, 0) || !nvfp4_ok(v4, 1)) return THRIFT_ERR_INVALID_ARG;
  if (outer <= 0 || Ncap <= 0 || len < 0 || T < 1 || (int64_t)len + T > Ncap) return THRIFT_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return THRIFT_ERR_UNSUPPORTED;
  if (block_k != 64 && block_k != 128) return THRIFT_ERR_UNSUPPORTED;
  if (Ncap % 128 != 0 || Ncap % block_k != 0) return THRIFT_ERR_UNSUPPORTED;
  if (outer * (int64_t)Ncap > (int64_t)INT32_MAX / 2) return THRIFT_ERR_UNSUPPORTED;
  for (const void* ptr : {k_new, v_new, (const void*)k, (const void*)v, (const void*)k4->codes,
                          (const void*)v4->codes})
    if (reinterpret_cast<uintptr_t>(ptr) % 16 != 0) return THRIFT_ERR_INVALID_ARG;
  return kv_append_launch(k_new, v_new, outer, Ncap, d, block_k, len, T, k, v, k4, v4, kbar,
                          static_cast<cudaStream_t>(stream));
}

thrift_status thrift_reset_device_status(void* ws, void* stream) {
  if (!ws || reinterpret_cast<uintptr_t>(ws) % 256 != 0) return THRIFT_ERR_WORKSPACE;
  return cudaMemsetAsync(ws, 0, kWsHeader, static_cast<cudaStream_t>(stream)) == cudaSuccess ? THRIFT_OK
                                                                                               : THRIFT_ERR_CUDA;
}

thrift_status thrift_get_device_status(const void* ws, void* stream, int32_t* status_out) {
  if (!ws || !status_out) return THRIFT_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, static_cast<const uint8_t*>(ws) + kWsStatusOff, sizeof(v), cudaMemcpyDeviceToHost, s) !=
      cudaSuccess)
    return THRIFT_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return THRIFT_ERR_CUDA;
  *status_out = v;
  return THRIFT_OK;
}

thrift_status thrift_debug_wait_timeout(void* ws, int64_t limit_cycles, void* stream) {
  if (!ws || reinterpret_cast<uintptr_t>(ws) % 256 != 0) return THRIFT_ERR_WORKSPACE;
  if (limit_cycles <= 0 || limit_cycles > (int64_t)1 << 34) return THRIFT_ERR_INVALID_ARG;
  return wait_timeout_launch(status_ptr(ws), limit_cycles, static_cast<cudaStream_t>(stream));
}

thrift_status thrift_debug_ex2(const float* x, float* y, int64_t n, int32_t which, void* stream) {
  if (!x || !y || n < 0 || (which != 0 && which != 1)) return THRIFT_ERR_INVALID_ARG;
  if (n == 0) return THRIFT_OK;
  return ex2_probe_launch(x, y, n, which, static_cast<cudaStream_t>(stream));
}

size_t thrift_debug_pipe_rates_ws_bytes(void) { return pipe_rates_ws_bytes(); }

thrift_status thrift_debug_pipe_rates(void* ws, size_t ws_bytes, double* out, void* stream) {
  if (!out) return THRIFT_ERR_INVALID_ARG;
  if (!ws_ok(ws, ws_bytes, pipe_rates_ws_bytes())) return THRIFT_ERR_WORKSPACE;
  return pipe_rates_launch(ws, out, static_cast<cudaStream_t>(stream));
}

int32_t thrift_debug_checks_enabled(void) {
#ifdef THRIFT_CHECKS
  return 1;
#else
  return 0;
#endif
}

thrift_status thrift_debug_check(void* ws, int32_t fail, void* stream) {
  if (!ws || reinterpret_cast<uintptr_t>(ws) % 256 != 0) return THRIFT_ERR_WORKSPACE;
  return check_probe_launch(status_ptr(ws), fail, static_cast<cudaStream_t>(stream));
}

const char* thrift_status_str(thrift_status s) {
  switch (s) {
    case THRIFT_OK: return "ok";
    case THRIFT_ERR_INVALID_ARG: return "invalid argument";
    case THRIFT_ERR_UNSUPPORTED: return "unsupported configuration";
    case THRIFT_ERR_CUDA: return "CUDA error";
    case THRIFT_ERR_TIMEOUT: return "device wait timed out";
    case THRIFT_ERR_WORKSPACE: return "workspace null, misaligned or too small";
    case THRIFT_ERR_CHECK: return "in-kernel bounds check failed";
  }
  return "unknown status";
}

}  // extern "C"
