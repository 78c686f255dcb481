// Activation quantizers that feed the block-scaled GEMMs: bf16 -> E4M3 with
// one fp32 scale per row (the W4A8 activations), and bf16 -> NVFP4 (e2m1
// codes, an E4M3 scale per 16 elements, one fp32 scale per tensor; the W4A4
// activations).
//
// The W4A8 and W4A4 combinations are listed on the Humming news page
// (section "one library, many formats"); the scale / zero-point parameters
// are part of the quantization description ("Humming: open-source kernel
// library for quantized inference", summary paragraph 2).  The rounding
// rules follow the OCP FP8 and MX specifications (round to nearest even,
// saturating to the largest finite value); every step is fp32 so the codes
// are reproducible bit for bit:
//   FP8 rows : s = amax/448 (1 for an all-zero row), q = RNE_E4M3(x / s)
//   NVFP4    : g = amax_tensor/2688 (1 for an all-zero tensor),
//              sb = RNE_E4M3(amax_block / (6*g)), d = E4M3(sb) * g,
//              c = RNE_e2m1(x / d) (0 when d == 0)
// A zero result is always written as +0 (code 0), never -0.
// HBM-bound elementwise kernels: coalesced 16-byte loads, grid sized in
// multiples of the SM count.
#include <cuda_bf16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <cuda_fp16.h>

#include <algorithm>

#include "hq_internal.h"
#include "ptx.cuh"

namespace hq {

namespace {

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint8_t e4m3_rne(float x) {
  uint8_t c = (uint8_t)__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
  return c == 0x80 ? 0 : c;
}
__device__ __forceinline__ float e4m3_value(uint8_t c) {
  __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)c, __NV_E4M3);
  return __half2float(__half(h));
}
__device__ __forceinline__ uint32_t e2m1_rne(float x) {
  uint32_t c = (uint32_t)__nv_cvt_float_to_fp4(x, __NV_E2M1, cudaRoundNearest) & 0xF;
  return (c & 7) == 0 ? 0 : c;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// One CTA per row: amax, then the per-row E4M3 quantization.
__global__ void fp8_rows_kernel(const uint4* __restrict__ x, int k_vec, uint2* __restrict__ q,
                                float* __restrict__ scale) {
  __shared__ float red[32];
  const uint4* row = x + (size_t)blockIdx.x * k_vec;
  float m = 0.f;
  for (int i = threadIdx.x; i < k_vec; i += blockDim.x) {
    const uint4 v = row[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) m = fmaxf(m, fmaxf(fabsf(bf16_lo(w[j])), fabsf(bf16_hi(w[j]))));
  }
  m = warp_max(m);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    v = warp_max(v);
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  const float amax = red[0];
  const float s = amax > 0.f ? amax / 448.f : 1.f;
  if (threadIdx.x == 0) scale[blockIdx.x] = s;
  uint2* qrow = q + (size_t)blockIdx.x * k_vec;
  for (int i = threadIdx.x; i < k_vec; i += blockDim.x) {
    const uint4 v = row[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t out[2] = {0, 0};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t lo = e4m3_rne(bf16_lo(w[j]) / s), hi = e4m3_rne(bf16_hi(w[j]) / s);
      out[j >> 1] |= (lo | (hi << 8)) << (16 * (j & 1));
    }
    qrow[i] = make_uint2(out[0], out[1]);
  }
}

// Per-CTA maxima of |x| over the whole tensor (first pass of NVFP4).
__global__ void amax_kernel(const uint4* __restrict__ x, size_t n_vec, float* __restrict__ block_max) {
  __shared__ float red[32];
  float m = 0.f;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_vec; i += (size_t)gridDim.x * blockDim.x) {
    const uint4 v = x[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) m = fmaxf(m, fmaxf(fabsf(bf16_lo(w[j])), fabsf(bf16_hi(w[j]))));
  }
  m = warp_max(m);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    v = warp_max(v);
    if (threadIdx.x == 0) block_max[blockIdx.x] = v;
  }
}

// One thread per 16-element block.  Every CTA re-reduces the per-CTA maxima
// of the first pass (a few hundred floats) to get the tensor amax.
__global__ void nvfp4_kernel(const uint4* __restrict__ x, size_t n_blocks, const float* __restrict__ block_max,
                             int n_max, uint2* __restrict__ codes, uint8_t* __restrict__ sf, float* __restrict__ g_out) {
  __shared__ float red[32];
  __shared__ float s_g;
  float m = 0.f;
  for (int i = threadIdx.x; i < n_max; i += blockDim.x) m = fmaxf(m, block_max[i]);
  m = warp_max(m);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    v = warp_max(v);
    if (threadIdx.x == 0) s_g = v > 0.f ? v / 2688.f : 1.f;
  }
  __syncthreads();
  const float g = s_g;
  if (blockIdx.x == 0 && threadIdx.x == 0) *g_out = g;
  const float six_g = 6.f * g;
  for (size_t b = (size_t)blockIdx.x * blockDim.x + threadIdx.x; b < n_blocks; b += (size_t)gridDim.x * blockDim.x) {
    const uint4 v0 = x[2 * b], v1 = x[2 * b + 1];
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    float f[16];
    float bmax = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      f[2 * j] = bf16_lo(w[j]);
      f[2 * j + 1] = bf16_hi(w[j]);
      bmax = fmaxf(bmax, fmaxf(fabsf(f[2 * j]), fabsf(f[2 * j + 1])));
    }
    const uint8_t sb = e4m3_rne(bmax / six_g);
    const float d = e4m3_value(sb) * g;
    uint32_t out[2] = {0, 0};
    if (d > 0.f) {
#pragma unroll
      for (int j = 0; j < 16; ++j) out[j >> 3] |= e2m1_rne(f[j] / d) << (4 * (j & 7));
    }
    codes[b] = make_uint2(out[0], out[1]);
    sf[b] = sb;
  }
}

}  // namespace

size_t nvfp4_quant_ws_bytes(int rows, int k) {
  (void)rows;
  (void)k;
  DeviceInfo dev{};
  int sms = device_info(&dev) == HQ_OK ? dev.num_sms : 148;
  return kWsScratchOff + (size_t)sms * 4 * sizeof(float);
}

hq_status fp8_rows_launch(const void* x, int rows, int k, void* q, float* scale, cudaStream_t s) {
  fp8_rows_kernel<<<rows, 256, 0, s>>>(static_cast<const uint4*>(x), k / 8, static_cast<uint2*>(q), scale);
  return cudaGetLastError() == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}

hq_status nvfp4_quant_launch(const void* x, int rows, int k, void* codes, void* sf, float* g, void* ws,
                             cudaStream_t s) {
  DeviceInfo dev{};
  device_info(&dev);
  const int grid = dev.num_sms * 4;
  float* block_max = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + kWsScratchOff);
  const size_t n = (size_t)rows * k;
  amax_kernel<<<grid, 256, 0, s>>>(static_cast<const uint4*>(x), n / 8, block_max);
  nvfp4_kernel<<<grid, 256, 0, s>>>(static_cast<const uint4*>(x), n / 16, block_max, grid, static_cast<uint2*>(codes),
                                    static_cast<uint8_t*>(sf), g);
  return cudaGetLastError() == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}

}  // namespace hq
