// Measured pipe rates for the elementwise bound of the attention kernel: lanes of ex2.approx.f32
// (the MUFU unit) and of fma.rn.f32 (the FMA pipe) completed per SM clock, with one CTA of 512
// threads per SM running eight independent chains per thread.
#include <cuda_runtime.h>

#include "sm100.cuh"
#include "thrift_internal.h"

namespace thrift {

namespace {

constexpr int kProbeThreads = 512;
constexpr int kProbeIters = 1024;

template <int WHICH>
__global__ void __launch_bounds__(kProbeThreads, 1) pipe_rate_kernel(unsigned long long* cycles, float* sink) {
  float a[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) a[i] = (float)((threadIdx.x + 3 * i) & 63) * 1e-3f - 0.03f;
  __syncthreads();
  const long long t0 = clock64();
  for (int it = 0; it < kProbeIters; ++it) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (WHICH == 0)
        asm volatile("ex2.approx.ftz.f32 %0, %0;" : "+f"(a[i]));
      else
        asm volatile("fma.rn.f32 %0, %0, 0f3F7FF972, 0f3A83126F;" : "+f"(a[i]));
    }
  }
  __syncthreads();
  const long long t1 = clock64();
  float s = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) s += a[i];
  if (s == 1234.5f) sink[threadIdx.x] = s;  // keeps the chains live
  if (threadIdx.x == 0) atomicMax(cycles + WHICH, (unsigned long long)(t1 - t0));
}

__global__ void pipe_rate_finish(const unsigned long long* cycles, double* out) {
  const double lanes = (double)kProbeThreads * kProbeIters * 8;
  out[0] = cycles[0] ? lanes / (double)cycles[0] : 0.0;
  out[1] = cycles[1] ? lanes / (double)cycles[1] : 0.0;
}

}  // namespace

thrift_status pipe_rates_launch(void* ws, double* out, cudaStream_t stream) {
  unsigned long long* cycles = reinterpret_cast<unsigned long long*>(static_cast<uint8_t*>(ws) + kWsHeader);
  float* sink = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + kWsHeader + 64);
  if (cudaMemsetAsync(cycles, 0, 2 * sizeof(unsigned long long), stream) != cudaSuccess) return THRIFT_ERR_CUDA;
  const int grid = num_sms();
  pipe_rate_kernel<0><<<grid, kProbeThreads, 0, stream>>>(cycles, sink);
  pipe_rate_kernel<1><<<grid, kProbeThreads, 0, stream>>>(cycles, sink);
  pipe_rate_finish<<<1, 1, 0, stream>>>(cycles, out);
  return cudaPeekAtLastError() == cudaSuccess ? THRIFT_OK : THRIFT_ERR_CUDA;
}

size_t pipe_rates_ws_bytes() { return kWsHeader + 64 + kProbeThreads * sizeof(float); }

__global__ void check_probe_kernel(int* status, int fail) {
  if (!THRIFT_CHECK(fail == 0, status)) return;
}

thrift_status check_probe_launch(int* status, int fail, cudaStream_t stream) {
  check_probe_kernel<<<1, 1, 0, stream>>>(status, fail);
  return cudaPeekAtLastError() == cudaSuccess ? THRIFT_OK : THRIFT_ERR_CUDA;
}

}  // namespace thrift
