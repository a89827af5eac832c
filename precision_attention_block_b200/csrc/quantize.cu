// NVFP4 quantisation of FP16 tensors (ThriftAttention technical summary, "FP4-pad": the NVFP4
// microscaling format -- E2M1 values, one E4M3 scale per 16 elements, one FP32 tensor scale).
//
// Two HBM-bound passes:
//   1. amax: every thread max-reduces 16-byte vectors of |x|, warp shuffles, one atomicMax per
//      block on the float bits (non-negative floats order like unsigned ints).
//   2. encode: per 16-element group s_b = E4M3(amax16 / 6 / s_t), codes = E2M1(x / (s_b s_t)),
//      with IEEE divisions (round to nearest) so that codes and scales are bit-identical to any
//      other correctly rounded implementation of the same steps.
//      Groups along d (Q, K): one thread per group, 32-byte loads, 8-byte code stores.
//      Groups along tokens (V): a 128-token x d tile is staged in shared memory and transposed.
// Inputs may be strided ([B, H, N, d] with any row strides, e.g. a token-major [B, N, H, d]
// tensor); the codes and scales are always written in the dense layouts.
#include <cuda_runtime.h>

#include "sm100.cuh"
#include "thrift_internal.h"

namespace thrift {

namespace {

__global__ void __launch_bounds__(256) amax_kernel(const uint4* __restrict__ x, int64_t n_vec,
                                                   unsigned int* __restrict__ amax_bits) {
  __half2 m2 = __float2half2_rn(0.0f);
  int64_t stride = (int64_t)gridDim.x * blockDim.x;
  int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (; i + 3 * stride < n_vec; i += 4 * stride) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = __ldg(x + i + u * stride);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const __half2* h = reinterpret_cast<const __half2*>(&v[u]);
#pragma unroll
      for (int t = 0; t < 4; ++t) m2 = __hmax2(m2, __habs2(h[t]));
    }
  }
  for (; i < n_vec; i += stride) {
    uint4 v = __ldg(x + i);
    const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
    for (int t = 0; t < 4; ++t) m2 = __hmax2(m2, __habs2(h[t]));
  }
  float m = fmaxf(__low2float(m2), __high2float(m2));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float red[8];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (threadIdx.x == 0) atomicMax(amax_bits, __float_as_uint(m));
  }
}

// amax of a strided tensor: CTA (tile, o) reads rows [64 tile, 64 tile + 64) of slice o.
__global__ void __launch_bounds__(256) amax_rows_kernel(const __half* __restrict__ x, RowMap rows, int N, int d,
                                                        unsigned int* __restrict__ amax_bits) {
  const int o = blockIdx.y, n0 = blockIdx.x * 64;
  const int d8 = d >> 3;
  const __half* base = x + rows.base(o);
  __half2 m2 = __float2half2_rn(0.0f);
  for (int v = threadIdx.x; v < 64 * d8; v += 256) {
    const int n = n0 + v / d8, c8 = v % d8;
    if (n >= N) break;
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(base + (int64_t)n * rows.sn + c8 * 8));
    const __half2* h = reinterpret_cast<const __half2*>(&w);
#pragma unroll
    for (int t = 0; t < 4; ++t) m2 = __hmax2(m2, __habs2(h[t]));
  }
  float m = fmaxf(__low2float(m2), __high2float(m2));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  __shared__ float red[8];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = threadIdx.x < 8 ? red[threadIdx.x] : 0.0f;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (threadIdx.x == 0) atomicMax(amax_bits, __float_as_uint(m));
  }
}

__device__ __forceinline__ float tensor_scale_from(unsigned int amax_bits) {
  float amax = __uint_as_float(amax_bits);
  return amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f;
}

// Quantise one group of 16 values; returns the E4M3 scale code, writes 8 code bytes.
__device__ __forceinline__ uint32_t quant16(const float (&x)[16], float s_t, uint2& packed) {
  float amax16 = 0.0f;
#pragma unroll
  for (int t = 0; t < 16; ++t) amax16 = fmaxf(amax16, fabsf(x[t]));
  float r = __fdiv_rn(amax16, 6.0f);
  uint32_t sb = cvt_e4m3(__fdiv_rn(r, s_t));
  float eff = __fmul_rn(e4m3_to_f32(sb), s_t);
  uint32_t w[2] = {0u, 0u};
  if (eff != 0.0f) {
#pragma unroll
    for (int t = 0; t < 16; t += 2) {
      uint32_t b = cvt_e2m1x2(__fdiv_rn(x[t], eff), __fdiv_rn(x[t + 1], eff));
      w[t >> 3] |= b << ((t & 7) * 4);
    }
  }
  packed = make_uint2(w[0], w[1]);
  return sb;
}

__device__ __forceinline__ int64_t sf_mma_offset(int64_t row, int64_t group, int64_t n_kblocks) {
  int64_t rb = row >> 7, kb = group >> 2;
  return (rb * n_kblocks + kb) * 512 + (row & 31) * 16 + ((row & 127) >> 5) * 4 + (group & 3);
}

// Groups along d: one thread per group of 16 consecutive elements of a row (group g of the dense
// order: row g / (d/16) = o * N + n; DENSE reads it at 16 g, otherwise through the row map).
template <bool DENSE>
__global__ void __launch_bounds__(256) encode_rows_kernel(const __half* __restrict__ xh, RowMap rows, int N,
                                                          int64_t n_groups, int d,
                                                          const unsigned int* __restrict__ amax_bits,
                                                          uint2* __restrict__ codes, uint8_t* __restrict__ scales,
                                                          uint8_t* __restrict__ scales_mma,
                                                          float* __restrict__ tensor_scale) {
  float s_t = tensor_scale_from(*amax_bits);
  if (blockIdx.x == 0 && threadIdx.x == 0) *tensor_scale = s_t;
  int gpr = d >> 4;  // groups per row
  int64_t n_kblocks = d >> 6;
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < n_groups;
       g += (int64_t)gridDim.x * blockDim.x) {
    const uint4* src;
    if constexpr (DENSE) {
      src = reinterpret_cast<const uint4*>(xh) + 2 * g;
    } else {
      const int64_t r = g / gpr;
      const int o = (int)(r / N), n = (int)(r - (int64_t)o * N);
      src = reinterpret_cast<const uint4*>(xh + rows.off(o, n) + (g - r * gpr) * 16);
    }
    uint4 v0 = __ldg(src), v1 = __ldg(src + 1);
    float f[16];
    const __half2* h0 = reinterpret_cast<const __half2*>(&v0);
    const __half2* h1 = reinterpret_cast<const __half2*>(&v1);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      float2 a = __half22float2(h0[t]), b = __half22float2(h1[t]);
      f[2 * t] = a.x; f[2 * t + 1] = a.y; f[8 + 2 * t] = b.x; f[8 + 2 * t + 1] = b.y;
    }
    uint2 packed;
    uint32_t sb = quant16(f, s_t, packed);
    codes[g] = packed;
    scales[g] = (uint8_t)sb;
    int64_t row = g / gpr;
    int64_t grp = g - row * gpr;
    scales_mma[sf_mma_offset(row, grp, n_kblocks)] = (uint8_t)sb;
  }
}

// Groups along tokens: one CTA per (outer index, 128-token tile); 256 threads.  The tile is staged
// in shared memory; thread (c, part) quantises channel c's GPT consecutive 16-token groups, so
// its codes (8 bytes per group), scales and tensor-core scales (one byte per group, consecutive
// in both layouts) leave as one contiguous store each instead of one per group.
template <int D>
__global__ void __launch_bounds__(256) encode_cols_kernel(const __half* __restrict__ x, RowMap rows, int N,
                                                          const unsigned int* __restrict__ amax_bits,
                                                          uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                                                          uint8_t* __restrict__ scales_mma,
                                                          float* __restrict__ tensor_scale) {
  constexpr int TOK = 128;
  constexpr int PARTS = 256 / D;           // token parts per channel
  constexpr int GPT = TOK / 16 / PARTS;    // groups per thread: 4 (D = 128) or 2 (D = 64)
  __shared__ __align__(16) __half tile[TOK * D];
  const float s_t = tensor_scale_from(*amax_bits);
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *tensor_scale = s_t;
  const int64_t o = blockIdx.y;
  const int t0 = blockIdx.x * TOK;
  const __half* src = x + rows.off((int)o, t0);
  uint4* dst = reinterpret_cast<uint4*>(tile);
  constexpr int VECS = TOK * D / 8;
#pragma unroll
  for (int v = threadIdx.x; v < VECS; v += 256)
    dst[v] = __ldg(reinterpret_cast<const uint4*>(src + (int64_t)(v / (D / 8)) * rows.sn + (v % (D / 8)) * 8));
  __syncthreads();
  const int c = threadIdx.x % D, part = threadIdx.x / D;
  const int g_first = part * GPT;  // first group of the thread within the tile
  uint32_t cw[2 * GPT];
  uint32_t sbs = 0;
#pragma unroll
  for (int gi = 0; gi < GPT; ++gi) {
    const int g = g_first + gi;
    float f[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) f[t] = __half2float(tile[(g * 16 + t) * D + c]);
    uint2 packed;
    const uint32_t sb = quant16(f, s_t, packed);
    cw[2 * gi] = packed.x;
    cw[2 * gi + 1] = packed.y;
    sbs |= sb << (8 * gi);
  }
  const int64_t row = o * D + c;
  const int64_t grp0 = (t0 >> 4) + g_first;  // a multiple of GPT
  uint8_t* cdst = codes + row * (N / 2) + grp0 * 8;
  if constexpr (GPT == 4) {
    reinterpret_cast<uint4*>(cdst)[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
    reinterpret_cast<uint4*>(cdst)[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
    *reinterpret_cast<uint32_t*>(scales + row * (N / 16) + grp0) = sbs;
    *reinterpret_cast<uint32_t*>(scales_mma + sf_mma_offset(row, grp0, N >> 6)) = sbs;
  } else {
    reinterpret_cast<uint4*>(cdst)[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
    *reinterpret_cast<uint16_t*>(scales + row * (N / 16) + grp0) = (uint16_t)sbs;
    *reinterpret_cast<uint16_t*>(scales_mma + sf_mma_offset(row, grp0, N >> 6)) = (uint16_t)sbs;
  }
}

__global__ void tensor_scale_kernel(const unsigned int* __restrict__ amax_bits, float* __restrict__ tensor_scale) {
  *tensor_scale = tensor_scale_from(*amax_bits);
}

// ---- appending to a double-cached KV cache (capacity Ncap, `len` keys held, T new keys)

// The T new rows of every (batch, KV head) into the FP16 cache at [len, len + T).
__global__ void __launch_bounds__(256) kv_copy_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, int T,
                                                      int Ncap, int len, int d8, int64_t total) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / d8, c = i - row * d8;
    const int64_t o = row / T, t = row - o * T;
    dst[(o * Ncap + len + t) * d8 + c] = src[i];
  }
}

// NVFP4 codes of the new K rows (groups along d) with the cache's fixed tensor scale.
__global__ void __launch_bounds__(256) kv_encode_rows_kernel(const __half* __restrict__ k, int Ncap, int len, int T,
                                                             int d, int64_t n_groups,
                                                             const float* __restrict__ tensor_scale,
                                                             uint2* __restrict__ codes, uint8_t* __restrict__ scales,
                                                             uint8_t* __restrict__ scales_mma) {
  const float s_t = __ldg(tensor_scale);
  const int gpr = d >> 4;
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < n_groups;
       g += (int64_t)gridDim.x * blockDim.x) {
    const int64_t rn = g / gpr, grp = g - rn * gpr;
    const int64_t o = rn / T, t = rn - o * T;
    const int64_t row = o * Ncap + len + t;
    const uint4* src = reinterpret_cast<const uint4*>(k + row * d + grp * 16);
    const uint4 v0 = __ldg(src), v1 = __ldg(src + 1);
    float f[16];
    const __half2* h0 = reinterpret_cast<const __half2*>(&v0);
    const __half2* h1 = reinterpret_cast<const __half2*>(&v1);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 a = __half22float2(h0[e]), b = __half22float2(h1[e]);
      f[2 * e] = a.x; f[2 * e + 1] = a.y; f[8 + 2 * e] = b.x; f[8 + 2 * e + 1] = b.y;
    }
    uint2 packed;
    const uint32_t sb = quant16(f, s_t, packed);
    codes[row * gpr + grp] = packed;
    scales[row * gpr + grp] = (uint8_t)sb;
    scales_mma[sf_mma_offset(row, grp, d >> 6)] = (uint8_t)sb;
  }
}

// NVFP4 codes of the 16-token V groups g0 .. g0 + ng - 1 (groups along tokens), from the FP16
// cache (zero past the keys held) with the cache's fixed tensor scale.
__global__ void __launch_bounds__(256) kv_encode_cols_kernel(const __half* __restrict__ v, int Ncap, int d, int g0,
                                                             int ng, int64_t total,
                                                             const float* __restrict__ tensor_scale,
                                                             uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                                                             uint8_t* __restrict__ scales_mma) {
  const float s_t = __ldg(tensor_scale);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t c = i % d, rest = i / d;
    const int64_t gi = rest % ng, o = rest / ng;
    const int64_t grp = g0 + gi;
    float f[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) f[t] = __half2float(v[(o * Ncap + grp * 16 + t) * d + c]);
    uint2 packed;
    const uint32_t sb = quant16(f, s_t, packed);
    const int64_t row = o * d + c;
    *reinterpret_cast<uint2*>(codes + row * (Ncap / 2) + grp * 8) = packed;
    scales[row * (Ncap / 16) + grp] = (uint8_t)sb;
    scales_mma[sf_mma_offset(row, grp, Ncap >> 6)] = (uint8_t)sb;
  }
}

// Means of the key blocks j0 .. j0 + nj - 1 over the keys each holds (below n_valid): exact FP16
// sums in float64 divided by the count.
__global__ void __launch_bounds__(256) kv_means_kernel(const __half* __restrict__ k, int Ncap, int d, int bk, int j0,
                                                       int nj, int n_valid, int64_t total, double* __restrict__ kbar) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t c = i % d, rest = i / d;
    const int64_t jj = rest % nj, o = rest / nj;
    const int64_t j = j0 + jj;
    const int cnt = (int)min((int64_t)bk, (int64_t)n_valid - j * bk);
    double s = 0.0;
    for (int t = 0; t < cnt; ++t) s += (double)__half2float(k[(o * Ncap + j * bk + t) * d + c]);
    kbar[(o * (Ncap / bk) + j) * d + c] = s / (double)cnt;
  }
}

}  // namespace

thrift_status tensor_scale_launch(const void* x, int64_t n, float* tensor_scale, unsigned int* amax_slot,
                                  cudaStream_t stream) {
  if (cudaMemsetAsync(amax_slot, 0, sizeof(unsigned int), stream) != cudaSuccess) return THRIFT_ERR_CUDA;
  int64_t blocks = (n / 8 + 4 * 256 - 1) / (4 * 256);
  if (blocks > (int64_t)num_sms() * 8) blocks = (int64_t)num_sms() * 8;
  if (blocks < 1) blocks = 1;
  amax_kernel<<<(unsigned)blocks, 256, 0, stream>>>(reinterpret_cast<const uint4*>(x), n / 8, amax_slot);
  tensor_scale_kernel<<<1, 1, 0, stream>>>(amax_slot, tensor_scale);
  return cudaPeekAtLastError() == cudaSuccess ? THRIFT_OK : THRIFT_ERR_CUDA;
}

thrift_status kv_append_launch(const void* k_new, const void* v_new, int64_t outer, int32_t Ncap, int32_t d,
                               int32_t block_k, int32_t len, int32_t T, void* k, void* v, const thrift_nvfp4* k4,
                               const thrift_nvfp4* v4, double* kbar, cudaStream_t stream) {
  const int sms = num_sms();
  auto grid_for = [&](int64_t work) {
    int64_t b = (work + 255) / 256;
    if (b > (int64_t)sms * 16) b = (int64_t)sms * 16;
    return (unsigned)(b < 1 ? 1 : b);
  };
  const int64_t vecs = outer * (int64_t)T * (d / 8);
  if (k_new) kv_copy_kernel<<<grid_for(vecs), 256, 0, stream>>>(reinterpret_cast<const uint4*>(k_new),
                                                                 reinterpret_cast<uint4*>(k), T, Ncap, len, d / 8, vecs);
  if (v_new) kv_copy_kernel<<<grid_for(vecs), 256, 0, stream>>>(reinterpret_cast<const uint4*>(v_new),
                                                                 reinterpret_cast<uint4*>(v), T, Ncap, len, d / 8, vecs);
  const int64_t kgroups = outer * (int64_t)T * (d / 16);
  kv_encode_rows_kernel<<<grid_for(kgroups), 256, 0, stream>>>(
      reinterpret_cast<const __half*>(k), Ncap, len, T, d, kgroups, k4->tensor_scale,
      reinterpret_cast<uint2*>(k4->codes), k4->scales, k4->scales_mma);
  const int g0 = len / 16, g1 = (len + T - 1) / 16;
  const int64_t vwork = outer * (int64_t)(g1 - g0 + 1) * d;
  kv_encode_cols_kernel<<<grid_for(vwork), 256, 0, stream>>>(reinterpret_cast<const __half*>(v), Ncap, d, g0,
                                                            g1 - g0 + 1, vwork, v4->tensor_scale, v4->codes,
                                                            v4->scales, v4->scales_mma);
  const int j0 = len / block_k, j1 = (len + T - 1) / block_k;
  const int64_t mwork = outer * (int64_t)(j1 - j0 + 1) * d;
  kv_means_kernel<<<grid_for(mwork), 256, 0, stream>>>(reinterpret_cast<const __half*>(k), Ncap, d, block_k, j0,
                                                      j1 - j0 + 1, len + T, mwork, kbar);
  return cudaPeekAtLastError() == cudaSuccess ? THRIFT_OK : THRIFT_ERR_CUDA;
}

size_t scales_mma_bytes(int64_t outer, int32_t N, int32_t d, int32_t group_axis) {
  int64_t rows = group_axis == 0 ? outer * N : outer * d;
  int64_t len = group_axis == 0 ? d : N;
  int64_t nrb = (rows + 127) / 128;
  return (size_t)(nrb * (len / 64) * 512);
}

thrift_status quantize_launch(const void* x, const RowMap& rows, int64_t outer, int32_t N, int32_t d,
                              const thrift_nvfp4* out, unsigned int* amax_slot, cudaStream_t stream) {
  int64_t total = outer * (int64_t)N * d;
  const bool dense = rows.dense((int)(outer / rows.H), N, d);
  const __half* xh = reinterpret_cast<const __half*>(x);
  if (cudaMemsetAsync(amax_slot, 0, sizeof(unsigned int), stream) != cudaSuccess) return THRIFT_ERR_CUDA;
  int sms = num_sms();
  if (dense) {
    int64_t amax_blocks = (total / 8 + 4 * 256 - 1) / (4 * 256);  // about four vectors per thread
    if (amax_blocks > (int64_t)sms * 8) amax_blocks = (int64_t)sms * 8;
    if (amax_blocks < 1) amax_blocks = 1;
    amax_kernel<<<(unsigned)amax_blocks, 256, 0, stream>>>(reinterpret_cast<const uint4*>(x), total / 8, amax_slot);
  } else {
    amax_rows_kernel<<<dim3((N + 63) / 64, (unsigned)outer), 256, 0, stream>>>(xh, rows, N, d, amax_slot);
  }
  if (out->group_axis == 0) {
    int64_t groups = total / 16;
    int64_t blocks = (groups + 255) / 256;
    if (blocks > (int64_t)sms * 32) blocks = (int64_t)sms * 32;
    auto kern = dense ? encode_rows_kernel<true> : encode_rows_kernel<false>;
    kern<<<(unsigned)blocks, 256, 0, stream>>>(xh, rows, N, groups, d, amax_slot,
                                               reinterpret_cast<uint2*>(out->codes), out->scales, out->scales_mma,
                                               out->tensor_scale);
  } else {
    dim3 grid(N / 128, (unsigned)outer);
    if (d == 128)
      encode_cols_kernel<128><<<grid, 256, 0, stream>>>(xh, rows, N, amax_slot, out->codes, out->scales,
                                                         out->scales_mma, out->tensor_scale);
    else
      encode_cols_kernel<64><<<grid, 256, 0, stream>>>(xh, rows, N, amax_slot, out->codes, out->scales,
                                                        out->scales_mma, out->tensor_scale);
  }
  return cudaPeekAtLastError() == cudaSuccess ? THRIFT_OK : THRIFT_ERR_CUDA;
}

}  // namespace thrift
