// Host-side declarations shared by the library's translation units (not part of the C ABI).
#pragma once
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "../../include/thrift.h"

namespace thrift {

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Element offsets in an FP16 tensor viewed as [B, H, N, d] with strides (sb, sh, sn) in elements
// (the d elements of a token row contiguous): row n of slice o = b * H + h starts at off(o, n).
struct RowMap {
  int64_t sb, sh, sn;
  int H;
  __host__ __device__ __forceinline__ int64_t base(int o) const {
    return (int64_t)(o / H) * sb + (int64_t)(o % H) * sh;
  }
  __host__ __device__ __forceinline__ int64_t off(int o, int n) const { return base(o) + (int64_t)n * sn; }
  // the dense layout (sb only matters with more than one batch)
  bool dense(int B, int N, int d) const {
    return sn == d && sh == (int64_t)N * d && (B == 1 || sb == (int64_t)H * N * d);
  }
};
inline RowMap dense_rows(int H, int N, int d) {
  return RowMap{(int64_t)H * N * d, (int64_t)N * d, (int64_t)d, H};
}

int num_sms();

// Unique id of the calling thread's current CUDA context (cuCtxGetId), 0 when none is current or
// the driver cannot tell; per-device caches of context-bound values are keyed by it.
unsigned long long current_context_id();

// Workspace: [0, 256) status word and small scalars; then per-call scratch.
constexpr size_t kWsHeader = 256;
constexpr size_t kWsStatusOff = 0;    // int32 device status
constexpr size_t kWsAmaxOff = 16;     // uint32 amax bits for the quantiser

struct SelectLayout {
  size_t qbar_off, kbar_off, scores_off, topk_hist_off, bytes;
};
SelectLayout select_layout(const thrift_cfg& c);

size_t scales_mma_bytes(int64_t outer, int32_t N, int32_t d, int32_t group_axis);

// x: [outer, N, d] rows addressed through `rows` (rows.H divides outer into batch and head).
thrift_status quantize_launch(const void* x, const RowMap& rows, int64_t outer, int32_t N, int32_t d,
                              const thrift_nvfp4* out, unsigned int* amax_slot, cudaStream_t stream);

thrift_status tensor_scale_launch(const void* x, int64_t n, float* tensor_scale, unsigned int* amax_slot,
                                  cudaStream_t stream);

thrift_status kv_append_launch(const void* k_new, const void* v_new, int64_t outer, int32_t Ncap, int32_t d,
                               int32_t block_k, int32_t len, int32_t T, void* k, void* v, const thrift_nvfp4* k4,
                               const thrift_nvfp4* v4, double* kbar, cudaStream_t stream);

thrift_status select_launch(const void* q, const RowMap& qrows, const void* k, const RowMap& krows,
                            const thrift_cfg& c, uint32_t* mask, int32_t* counts, int16_t* lists, double* scores_out,
                            uint8_t* scratch, cudaStream_t stream);

size_t noalloc_select_scratch_bytes();
thrift_status noalloc_select_scratch(uint8_t** out);

// Row maps of the FP16 operands and of the output of one attention launch (dense unless given).
struct AttnRows {
  RowMap q, k, v, out;
};
AttnRows dense_attn_rows(const thrift_cfg& c);

// The fused attention launch.  mode: 0 = FP16 pairs from the mask, 1 = every pair NVFP4,
// 2 = every pair FP16, 3 = only the FP16 pairs of the mask (the compute-matched sparse variant; no
// NVFP4 operand is read).  out_hp: the FP32 copy of the output (may be null); running_max: the
// running maximum as the P requantisation's first level (reading R2); dbg, dbg_entry: the debug
// dump of one entry (null and -1 normally); rows: null for dense operands and output.
thrift_status attn_launch_dbg(const void* q, const void* k, const void* v, const thrift_nvfp4* q4,
                              const thrift_nvfp4* k4, const thrift_nvfp4* v4, const uint32_t* mask, int mode,
                              void* out, float* out_hp, float* lse, int running_max, const thrift_cfg& c, int* status,
                              float* dbg, int dbg_entry, cudaStream_t stream, const AttnRows* rows = nullptr);

thrift_status wait_timeout_launch(int* status, long long limit, cudaStream_t stream);

thrift_status pipe_rates_launch(void* ws, double* out, cudaStream_t stream);
thrift_status ex2_probe_launch(const float* x, float* y, int64_t n, int which, cudaStream_t stream);
size_t pipe_rates_ws_bytes();
thrift_status check_probe_launch(int* status, int fail, cudaStream_t stream);

// ---- decode
// The cache's valid length (thrift_decode_cfg.n_valid, 0 meaning the whole capacity).
inline int decode_valid(const thrift_decode_cfg& c) { return c.n_valid > 0 ? c.n_valid : c.Nk; }

struct DecodeArgs {
  const thrift_decode_cfg* cfg;
  const void *q, *k, *v;
  const thrift_nvfp4 *q4, *k4, *v4;  // q4: the query rows' NVFP4 copy (workspace)
  const uint32_t* mask;
  int mode;  // as attn_launch
  void* out;
  float* lse;
  float* part_o;   // [B*Hkv, n_split, 16, d]
  float* part_ml;  // [B*Hkv, n_split, 16, 2]
  int* status;
};

// Upper bound of the number of key-block splits of a decode step with nkb key blocks.
int decode_split_cap(int nkb);

thrift_status decode_attn_launch(const DecodeArgs& a, cudaStream_t stream);

thrift_status kv_means_launch(const void* k, int64_t outer, int32_t Nk, int32_t d, int32_t block_k, double* kbar,
                              cudaStream_t stream);

// Decode selection: scores [B*Hq, nkb] live in `scratch` (decode_select_scratch_bytes) unless
// scores_out is given; counts and lists are skipped when either is null.
size_t decode_select_scratch_bytes(const thrift_decode_cfg& c);
thrift_status decode_select_launch(const void* q, const double* kbar, const thrift_decode_cfg& c, uint32_t* mask,
                                   int32_t* counts, int16_t* lists, double* scores_out, uint8_t* scratch,
                                   cudaStream_t stream);

}  // namespace thrift
