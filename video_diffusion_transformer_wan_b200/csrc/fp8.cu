// E4M3 quantisation for the FP8 linear layers of the Wan 2.1 DiT block ("Wan: Open and
// Advanced Large-Scale Video Generative Models", section "Infra", inference
// optimisation: FP8 GEMM with a per-tensor scale for the weights and a per-token scale
// for the activations).
//
// Codes are q = round_to_nearest_even_satfinite(x / s) with s = amax / 448 (1 when the
// amax is 0); the division is an IEEE float32 division, so a code depends only on the
// float32 input and its scale.
//
// quantize_rows_kernel: one warp per row, 8 elements per lane per step (one 16-byte
//   load of bf16 or two of fp32); pass 1 takes the row's amax, pass 2 (served by L1/L2)
//   writes the codes. With sum_halves the row is x[:, :K] + x[:, K:2K] (the I2V text and
//   image attention outputs, summed before quantisation).
// amax_kernel + quantize_tensor_kernel + scale_kernel: one scale for a whole tensor
//   (weights; an offline step).
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace wan {
namespace {

template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&v)[8]);

template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 f = __bfloat1622float2(h[j]);
    v[2 * j] = f.x;
    v[2 * j + 1] = f.y;
  }
}
template <>
__device__ __forceinline__ void load8<float>(const float* p, float (&v)[8]) {
  const float4 a = reinterpret_cast<const float4*>(p)[0];
  const float4 b = reinterpret_cast<const float4*>(p)[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

template <typename T>
__device__ __forceinline__ void row8(const T* xr, int c, int K, bool sum_halves, float (&v)[8]) {
  load8<T>(xr + c, v);
  if (sum_halves) {
    float w[8];
    load8<T>(xr + K + c, w);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] += w[i];
  }
}

__device__ __forceinline__ float scale_of(float amax) { return amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f; }

__device__ __forceinline__ uint2 codes8(const float (&v)[8], float s) {
  uint2 c;
  c.x = pack_e4m3x4(__fdiv_rn(v[0], s), __fdiv_rn(v[1], s), __fdiv_rn(v[2], s), __fdiv_rn(v[3], s));
  c.y = pack_e4m3x4(__fdiv_rn(v[4], s), __fdiv_rn(v[5], s), __fdiv_rn(v[6], s), __fdiv_rn(v[7], s));
  return c;
}

template <typename T>
__global__ void __launch_bounds__(256) quantize_rows_kernel(const T* __restrict__ x, int64_t x_stride, int M, int K,
                                                            int sum_halves, uint8_t* __restrict__ q,
                                                            float* __restrict__ scale) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= M) return;
  const T* xr = x + static_cast<int64_t>(warp) * x_stride;
  float am = 0.f;
  for (int c = lane * 8; c < K; c += 256) {
    float v[8];
    row8<T>(xr, c, K, sum_halves != 0, v);
#pragma unroll
    for (int i = 0; i < 8; ++i) am = fmaxf(am, fabsf(v[i]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
  const float s = scale_of(am);
  if (lane == 0) scale[warp] = s;
  uint8_t* qr = q + static_cast<int64_t>(warp) * K;
  for (int c = lane * 8; c < K; c += 256) {
    float v[8];
    row8<T>(xr, c, K, sum_halves != 0, v);
    *reinterpret_cast<uint2*>(qr + c) = codes8(v, s);
  }
}

template <typename T>
__global__ void __launch_bounds__(256) amax_kernel(const T* __restrict__ x, int64_t n8, unsigned* __restrict__ amax) {
  float am = 0.f;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float v[8];
    load8<T>(x + i * 8, v);
#pragma unroll
    for (int j = 0; j < 8; ++j) am = fmaxf(am, fabsf(v[j]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
  // non-negative floats order like their bit patterns
  if ((threadIdx.x & 31) == 0) atomicMax(amax, __float_as_uint(am));
}

template <typename T>
__global__ void __launch_bounds__(256) quantize_tensor_kernel(const T* __restrict__ x, int64_t n8,
                                                              const unsigned* __restrict__ amax,
                                                              uint8_t* __restrict__ q) {
  const float s = scale_of(__uint_as_float(*amax));
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float v[8];
    load8<T>(x + i * 8, v);
    *reinterpret_cast<uint2*>(q + i * 8) = codes8(v, s);
  }
}

__global__ void scale_kernel(unsigned* amax_then_scale) {
  const float s = scale_of(__uint_as_float(*amax_then_scale));
  *reinterpret_cast<float*>(amax_then_scale) = s;
}

unsigned blocks_for(int64_t n, int per_block) {
  int64_t b = (n + per_block - 1) / per_block;
  if (b > 148 * 16) b = 148 * 16;
  return static_cast<unsigned>(b < 1 ? 1 : b);
}

}  // namespace

int launch_quantize_rows(const void* x, int64_t x_stride, int M, int K, bool sum_halves, void* q, float* scale,
                         int dtype, cudaStream_t s) {
  if (M == 0 || K == 0) return WAN_OK;
  if (K % 8 != 0 || x_stride % 8 != 0) return WAN_ERR_SHAPE;
  trace_launch_begin(WAN_KIND_SMALL, s,
                     static_cast<double>(M) * K * ((sum_halves ? 2.0 : 1.0) * dtype_size(dtype) + 1.0));
  const unsigned blocks = static_cast<unsigned>((static_cast<int64_t>(M) * 32 + 255) / 256);
  if (dtype == WAN_BF16)
    quantize_rows_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x), x_stride, M, K,
                                                               sum_halves ? 1 : 0, static_cast<uint8_t*>(q), scale);
  else
    quantize_rows_kernel<float><<<blocks, 256, 0, s>>>(static_cast<const float*>(x), x_stride, M, K,
                                                       sum_halves ? 1 : 0, static_cast<uint8_t*>(q), scale);
  const int st = check_launch();
  trace_launch_end(WAN_KIND_SMALL, s);
  return st;
}

int launch_quantize_tensor(const void* x, int64_t n, void* q, float* scale, int dtype, cudaStream_t s) {
  if (n == 0) return WAN_OK;
  if (n % 8 != 0) return WAN_ERR_SHAPE;
  unsigned* am = reinterpret_cast<unsigned*>(scale);
  if (cudaMemsetAsync(am, 0, sizeof(unsigned), s) != cudaSuccess) return WAN_ERR_CUDA;
  const int64_t n8 = n / 8;
  const unsigned blocks = blocks_for(n8, 256);
  if (dtype == WAN_BF16) {
    amax_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x), n8, am);
    quantize_tensor_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x), n8, am,
                                                                 static_cast<uint8_t*>(q));
  } else {
    amax_kernel<float><<<blocks, 256, 0, s>>>(static_cast<const float*>(x), n8, am);
    quantize_tensor_kernel<float><<<blocks, 256, 0, s>>>(static_cast<const float*>(x), n8, am,
                                                         static_cast<uint8_t*>(q));
  }
  scale_kernel<<<1, 1, 0, s>>>(am);
  count_launches(3);
  return check_launch();
}

}  // namespace wan
