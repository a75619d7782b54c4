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

// ---- 8-bit attention operands (q per (row, head); k and v per (sample, head)) ----

// One warp per (sample, query row, head): 128 elements, 4 per lane.
__global__ void __launch_bounds__(256) attn_q_quant_kernel(const __nv_bfloat16* __restrict__ q, int64_t row_stride,
                                                           int col0, int H, int64_t n_units,
                                                           uint8_t* __restrict__ codes, float* __restrict__ scale) {
  const int64_t u = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (u >= n_units) return;
  const int64_t row = u / H;
  const int h = static_cast<int>(u - row * H);
  const uint2 raw = *reinterpret_cast<const uint2*>(q + row * row_stride + col0 + h * 128 + lane * 4);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
  const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
  float am = fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(c.x), fabsf(c.y)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
  const float s = scale_of(am);
  *reinterpret_cast<uint32_t*>(codes + u * 128 + lane * 4) =
      pack_e4m3x4(__fdiv_rn(a.x, s), __fdiv_rn(a.y, s), __fdiv_rn(c.x, s), __fdiv_rn(c.y, s));
  if (lane == 0) scale[u] = s;
}

// amax of k and of v per (sample, head): block (row chunk, head, sample), 16 threads per
// 128-element row, 8 elements each.
constexpr int kKvAmaxRows = 512;
__global__ void __launch_bounds__(256) attn_kv_amax_kernel(const __nv_bfloat16* __restrict__ k, int64_t ks, int kc,
                                                           const __nv_bfloat16* __restrict__ v, int64_t vs, int vc,
                                                           int Lk, int H, unsigned* __restrict__ amax) {
  const int b = blockIdx.z, h = blockIdx.y;
  const int r0 = blockIdx.x * kKvAmaxRows;
  const int r1 = min(r0 + kKvAmaxRows, Lk);
  const int c = (threadIdx.x & 15) * 8;
  float ak = 0.f, av = 0.f;
  for (int r = r0 + (threadIdx.x >> 4); r < r1; r += 16) {
    const int64_t row = static_cast<int64_t>(b) * Lk + r;
    float x[8];
    load8<__nv_bfloat16>(k + row * ks + kc + h * 128 + c, x);
#pragma unroll
    for (int i = 0; i < 8; ++i) ak = fmaxf(ak, fabsf(x[i]));
    load8<__nv_bfloat16>(v + row * vs + vc + h * 128 + c, x);
#pragma unroll
    for (int i = 0; i < 8; ++i) av = fmaxf(av, fabsf(x[i]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ak = fmaxf(ak, __shfl_xor_sync(0xffffffffu, ak, o));
    av = fmaxf(av, __shfl_xor_sync(0xffffffffu, av, o));
  }
  if ((threadIdx.x & 31) == 0) {
    // non-negative floats order like their bit patterns
    atomicMax(&amax[2 * (b * H + h)], __float_as_uint(ak));
    atomicMax(&amax[2 * (b * H + h) + 1], __float_as_uint(av));
  }
}

// k codes: one thread per 8 elements of a (row, head).
__global__ void __launch_bounds__(256) attn_k_quant_kernel(const __nv_bfloat16* __restrict__ k, int64_t ks, int kc,
                                                           int Lk, int H, int64_t n8, const unsigned* __restrict__ amax,
                                                           uint8_t* __restrict__ codes) {
  for (int64_t g = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; g < n8;
       g += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = g / (H * 16);
    const int rem = static_cast<int>(g - row * (H * 16));
    const int h = rem >> 4, c = (rem & 15) * 8;
    const int b = static_cast<int>(row / Lk);
    const float s = scale_of(__uint_as_float(amax[2 * (b * H + h)]));
    float x[8];
    load8<__nv_bfloat16>(k + row * ks + kc + h * 128 + c, x);
    *reinterpret_cast<uint2*>(codes + row * (static_cast<int64_t>(H) * 128) + h * 128 + c) = codes8(x, s);
  }
}

// v^T codes: block (64-key chunk, head, sample). Thread (dim group g = tid % 16 of 8 dims,
// key group kg = tid / 16 of 4 keys) quantises a 4 x 8 block and keeps, per dim, the 4
// keys' codes as one word; the block then writes 128 dim rows of 64 codes. Keys past Lk
// get code 0.
__global__ void __launch_bounds__(256) attn_vt_quant_kernel(const __nv_bfloat16* __restrict__ v, int64_t vs, int vc,
                                                            int Lk, int H, const unsigned* __restrict__ amax,
                                                            uint8_t* __restrict__ vt, int64_t vt_stride) {
  __shared__ uint32_t tile[128][17];  // [dim][4-key word], padded
  const int b = blockIdx.z, h = blockIdx.y;
  const int key0 = blockIdx.x * 64;
  const int g = threadIdx.x & 15, kg = threadIdx.x >> 4;
  const float s = scale_of(__uint_as_float(amax[2 * (b * H + h) + 1]));
  float x[4][8];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int key = key0 + kg * 4 + r;
    if (key < Lk) {
      load8<__nv_bfloat16>(v + (static_cast<int64_t>(b) * Lk + key) * vs + vc + h * 128 + g * 8, x[r]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) x[r][i] = 0.f;
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i)
    tile[g * 8 + i][kg] = pack_e4m3x4(__fdiv_rn(x[0][i], s), __fdiv_rn(x[1][i], s), __fdiv_rn(x[2][i], s),
                                      __fdiv_rn(x[3][i], s));
  __syncthreads();
  const int d = threadIdx.x >> 1, part = threadIdx.x & 1;
  uint8_t* dst = vt + (static_cast<int64_t>(b * H + h) * 128 + d) * vt_stride + key0 + part * 32;
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const int w = part * 8 + q * 4;
    *reinterpret_cast<uint4*>(dst + q * 16) = make_uint4(tile[d][w], tile[d][w + 1], tile[d][w + 2], tile[d][w + 3]);
  }
}

__global__ void kv_scale_kernel(unsigned* amax_then_scale, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) reinterpret_cast<float*>(amax_then_scale)[i] = scale_of(__uint_as_float(amax_then_scale[i]));
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

int launch_attn_fp8_quantize(const void* q, int64_t q_row_stride, int q_col0, const void* k, int64_t k_row_stride,
                             int k_col0, const void* v, int64_t v_row_stride, int v_col0, int B, int H, int Lq, int Lk,
                             void* q_codes, float* q_scale, void* k_codes, void* vt_codes, int64_t vt_stride,
                             float* kv_scale, cudaStream_t s) {
  if (B == 0) return WAN_OK;
  if (Lk <= 0 || Lq < 0 || H <= 0) return WAN_ERR_SHAPE;
  if (q_row_stride % 8 || k_row_stride % 8 || v_row_stride % 8 || q_col0 % 8 || k_col0 % 8 || v_col0 % 8 ||
      vt_stride % 64 || vt_stride < Lk)
    return WAN_ERR_ALIGN;
  const auto* qb = static_cast<const __nv_bfloat16*>(q);
  const auto* kb = static_cast<const __nv_bfloat16*>(k);
  const auto* vb = static_cast<const __nv_bfloat16*>(v);
  unsigned* am = reinterpret_cast<unsigned*>(kv_scale);
  if (cudaMemsetAsync(am, 0, sizeof(unsigned) * 2 * B * H, s) != cudaSuccess) return WAN_ERR_CUDA;
  trace_launch_begin(WAN_KIND_SMALL, s,
                     (static_cast<double>(B) * (Lq + 3.0 * Lk) * H * 128) * 2 + static_cast<double>(B) * (Lq + 2.0 * Lk) * H * 128);
  attn_kv_amax_kernel<<<dim3((Lk + kKvAmaxRows - 1) / kKvAmaxRows, H, B), 256, 0, s>>>(kb, k_row_stride, k_col0, vb,
                                                                                       v_row_stride, v_col0, Lk, H, am);
  const int64_t q_units = static_cast<int64_t>(B) * Lq * H;
  if (q_units > 0)
    attn_q_quant_kernel<<<static_cast<unsigned>((q_units * 32 + 255) / 256), 256, 0, s>>>(
        qb, q_row_stride, q_col0, H, q_units, static_cast<uint8_t*>(q_codes), q_scale);
  const int64_t k8 = static_cast<int64_t>(B) * Lk * H * 16;
  attn_k_quant_kernel<<<blocks_for(k8, 256), 256, 0, s>>>(kb, k_row_stride, k_col0, Lk, H, k8, am,
                                                          static_cast<uint8_t*>(k_codes));
  attn_vt_quant_kernel<<<dim3((Lk + 63) / 64, H, B), 256, 0, s>>>(vb, v_row_stride, v_col0, Lk, H, am,
                                                                  static_cast<uint8_t*>(vt_codes), vt_stride);
  kv_scale_kernel<<<(2 * B * H + 255) / 256, 256, 0, s>>>(am, 2 * B * H);
  count_launches(q_units > 0 ? 4 : 3);  // five or four kernels, one counted by trace_launch_begin
  const int st = check_launch();
  trace_launch_end(WAN_KIND_SMALL, s);
  return st;
}

}  // namespace wan
