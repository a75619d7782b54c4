// Kernel (a): LayerNorm without affine parameters, fused with the AdaLN modulation
// h = LN(x) * (1 + scale) + shift of the Wan 2.1 DiT block ("Wan: Open and Advanced
// Large-Scale Video Generative Models", section "Diffusion Transformer": a shared MLP
// predicts six modulation vectors, each block adds its own bias).
//
// HBM-bound: per row it reads D fp32 and writes D outputs. TPR threads own a row; each
// thread holds NU units of 8 consecutive floats in registers (two 128-bit loads per
// unit, one 128-bit bf16 store), so the row is read from HBM exactly once. Mean and
// variance are two passes over the registers (warp shuffles, then shared memory when
// a row spans several warps).
#include <cuda_bf16.h>

#include "internal.h"

namespace wan {
namespace {

constexpr int kNormThreads = 256;

template <typename OutT>
__device__ __forceinline__ void store8(OutT* dst, const float (&v)[8]);

template <>
__device__ __forceinline__ void store8<__nv_bfloat16>(__nv_bfloat16* dst, const float (&v)[8]) {
  uint4 u;
  __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]);
  __nv_bfloat162 b = __floats2bfloat162_rn(v[2], v[3]);
  __nv_bfloat162 c = __floats2bfloat162_rn(v[4], v[5]);
  __nv_bfloat162 d = __floats2bfloat162_rn(v[6], v[7]);
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  u.z = *reinterpret_cast<uint32_t*>(&c);
  u.w = *reinterpret_cast<uint32_t*>(&d);
  *reinterpret_cast<uint4*>(dst) = u;
}
template <>
__device__ __forceinline__ void store8<float>(float* dst, const float (&v)[8]) {
  reinterpret_cast<float4*>(dst)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(dst)[1] = make_float4(v[4], v[5], v[6], v[7]);
}

template <int TPR>
__device__ __forceinline__ float row_sum(float v, float* red, int row_in_block, int t) {
  constexpr int W = TPR < 32 ? TPR : 32;
#pragma unroll
  for (int o = W / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o, W);
  if constexpr (TPR > 32) {
    constexpr int NW = TPR / 32;
    float* r = red + row_in_block * NW;
    __syncthreads();
    if ((t & 31) == 0) r[t >> 5] = v;
    __syncthreads();
    v = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) v += r[w];
  }
  return v;
}

template <int TPR, int NU, typename OutT>
__global__ void __launch_bounds__(kNormThreads) layernorm_mod_kernel(
    const float* __restrict__ x, int64_t rows, int D, int L, const float* __restrict__ e,
    const float* __restrict__ mod_bias, int chunk, OutT* __restrict__ out, float eps) {
  constexpr int RPB = kNormThreads / TPR;
  __shared__ float red[(TPR > 32) ? RPB * (TPR / 32) : 1];
  const int row_in_block = threadIdx.x / TPR;
  const int t = threadIdx.x % TPR;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * RPB + row_in_block;
  const bool active = row < rows;
  const float* xr = x + (active ? row : 0) * D;

  float v[NU][8];
#pragma unroll
  for (int u = 0; u < NU; ++u) {
    const int col = (u * TPR + t) * 8;
    const float4 a = __ldcs(reinterpret_cast<const float4*>(xr + col));
    const float4 b = __ldcs(reinterpret_cast<const float4*>(xr + col + 4));
    v[u][0] = a.x; v[u][1] = a.y; v[u][2] = a.z; v[u][3] = a.w;
    v[u][4] = b.x; v[u][5] = b.y; v[u][6] = b.z; v[u][7] = b.w;
  }
  float s = 0.f;
#pragma unroll
  for (int u = 0; u < NU; ++u)
#pragma unroll
    for (int i = 0; i < 8; ++i) s += v[u][i];
  const float mean = row_sum<TPR>(s, red, row_in_block, t) / static_cast<float>(D);
  float q = 0.f;
#pragma unroll
  for (int u = 0; u < NU; ++u)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float c = v[u][i] - mean;
      q += c * c;
    }
  const float var = row_sum<TPR>(q, red, row_in_block, t) / static_cast<float>(D);
  const float rstd = 1.0f / sqrtf(var + eps);
  if (!active) return;

  const float* shift = nullptr;
  const float* scale = nullptr;
  const float* bshift = nullptr;
  const float* bscale = nullptr;
  if (chunk >= 0) {
    const int64_t b = row / L;
    shift = e + (b * 6 + 3 * chunk) * D;
    scale = shift + D;
    if (mod_bias) {
      bshift = mod_bias + (3 * chunk) * D;
      bscale = bshift + D;
    }
  }
  OutT* orow = out + row * D;
#pragma unroll
  for (int u = 0; u < NU; ++u) {
    const int col = (u * TPR + t) * 8;
    float o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = (v[u][i] - mean) * rstd;
    if (chunk >= 0) {
      float sh[8], sc[8];
      *reinterpret_cast<float4*>(sh) = *reinterpret_cast<const float4*>(shift + col);
      *reinterpret_cast<float4*>(sh + 4) = *reinterpret_cast<const float4*>(shift + col + 4);
      *reinterpret_cast<float4*>(sc) = *reinterpret_cast<const float4*>(scale + col);
      *reinterpret_cast<float4*>(sc + 4) = *reinterpret_cast<const float4*>(scale + col + 4);
      if (bshift) {
        float bs[8], bc[8];
        *reinterpret_cast<float4*>(bs) = *reinterpret_cast<const float4*>(bshift + col);
        *reinterpret_cast<float4*>(bs + 4) = *reinterpret_cast<const float4*>(bshift + col + 4);
        *reinterpret_cast<float4*>(bc) = *reinterpret_cast<const float4*>(bscale + col);
        *reinterpret_cast<float4*>(bc + 4) = *reinterpret_cast<const float4*>(bscale + col + 4);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          sh[i] += bs[i];
          sc[i] += bc[i];
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = o[i] * (1.0f + sc[i]) + sh[i];
    }
    store8<OutT>(orow + col, o);
  }
}

// Generic fallback for widths without a register-resident instantiation: one block per
// row, reads the row twice (the second read is served by L1/L2).
template <typename OutT>
__global__ void __launch_bounds__(kNormThreads) layernorm_mod_generic(
    const float* __restrict__ x, int64_t rows, int D, int L, const float* __restrict__ e,
    const float* __restrict__ mod_bias, int chunk, OutT* __restrict__ out, float eps) {
  __shared__ float red[kNormThreads / 32];
  const int64_t row = blockIdx.x;
  const float* xr = x + row * D;
  auto block_sum = [&](float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    float r = 0.f;
    for (int w = 0; w < kNormThreads / 32; ++w) r += red[w];
    return r;
  };
  float s = 0.f;
  for (int c = threadIdx.x; c < D; c += kNormThreads) s += xr[c];
  const float mean = block_sum(s) / D;
  float q = 0.f;
  for (int c = threadIdx.x; c < D; c += kNormThreads) {
    const float d = xr[c] - mean;
    q += d * d;
  }
  const float rstd = 1.0f / sqrtf(block_sum(q) / D + eps);
  const int64_t b = row / L;
  for (int c = threadIdx.x; c < D; c += kNormThreads) {
    float o = (xr[c] - mean) * rstd;
    if (chunk >= 0) {
      float sh = e[(b * 6 + 3 * chunk) * D + c];
      float sc = e[(b * 6 + 3 * chunk + 1) * D + c];
      if (mod_bias) {
        sh += mod_bias[(3 * chunk) * D + c];
        sc += mod_bias[(3 * chunk + 1) * D + c];
      }
      o = o * (1.0f + sc) + sh;
    }
    out[row * D + c] = static_cast<OutT>(o);
  }
}

template <typename OutT, int TPR, int NU>
int launch_fixed(const float* x, int64_t rows, int D, int L, const float* e, const float* mb, int chunk,
                 OutT* out, float eps, cudaStream_t s) {
  constexpr int RPB = kNormThreads / TPR;
  const int64_t blocks = (rows + RPB - 1) / RPB;
  layernorm_mod_kernel<TPR, NU, OutT><<<static_cast<unsigned>(blocks), kNormThreads, 0, s>>>(
      x, rows, D, L, e, mb, chunk, out, eps);
  return check_launch();
}

template <typename OutT>
int launch_typed(const float* x, int64_t rows, int D, int L, const float* e, const float* mb, int chunk, OutT* out,
                 float eps, cudaStream_t s) {
  const int units = D / 8;
  if (D % 8 == 0) {
#define WAN_LN_CASE(TPR, NU) \
  if (units == (TPR) * (NU)) return launch_fixed<OutT, TPR, NU>(x, rows, D, L, e, mb, chunk, out, eps, s);
    WAN_LN_CASE(8, 1)
    WAN_LN_CASE(16, 1)
    WAN_LN_CASE(32, 1)
    WAN_LN_CASE(32, 2)
    WAN_LN_CASE(32, 3)
    WAN_LN_CASE(32, 4)
    WAN_LN_CASE(32, 5)
    WAN_LN_CASE(32, 6)
    WAN_LN_CASE(32, 7)
    WAN_LN_CASE(32, 8)
    WAN_LN_CASE(128, 3)
    WAN_LN_CASE(128, 4)
    WAN_LN_CASE(128, 5)
    WAN_LN_CASE(128, 6)
    WAN_LN_CASE(128, 7)
    WAN_LN_CASE(128, 8)
#undef WAN_LN_CASE
  }
  layernorm_mod_generic<OutT><<<static_cast<unsigned>(rows), kNormThreads, 0, s>>>(x, rows, D, L, e, mb, chunk,
                                                                                     out, eps);
  return check_launch();
}

}  // namespace

int launch_layernorm(const float* x, int64_t rows, int D, int L, const float* e, const float* mod_bias, int chunk,
                     void* out, int dtype, float eps, cudaStream_t s) {
  if (rows == 0) return WAN_OK;
  // bytes: the fp32 row in, the row out (modulation vectors are L2-resident and excluded)
  trace_launch_begin(WAN_KIND_NORM, s, static_cast<double>(rows) * D * (4.0 + dtype_size(dtype)));
  int st = dtype == WAN_BF16
               ? launch_typed<__nv_bfloat16>(x, rows, D, L, e, mod_bias, chunk,
                                             static_cast<__nv_bfloat16*>(out), eps, s)
               : launch_typed<float>(x, rows, D, L, e, mod_bias, chunk, static_cast<float*>(out), eps, s);
  trace_launch_end(WAN_KIND_NORM, s);
  return st;
}

}  // namespace wan
