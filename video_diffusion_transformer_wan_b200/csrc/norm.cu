// Kernel (a): LayerNorm without affine parameters, fused with the AdaLN modulation
// h = LN(x) * (1 + scale) + shift of the Wan 2.1 DiT block ("Wan: Open and Advanced
// Large-Scale Video Generative Models", section "Diffusion Transformer": a shared MLP
// predicts six modulation vectors, each block adds its own bias).
//
// HBM-bound: per row it reads D fp32 and writes D outputs, i.e. 6 bytes per element
// for a bf16 output. A row group of TPR threads owns one row at a time; each thread
// holds NU units of 8 consecutive floats (two 128-bit loads, one 128-bit bf16 store).
// The kernel is persistent: a row group walks rows with a grid-wide stride, keeps its
// slice of shift and (1 + scale) in registers for as long as the sample does not
// change (so modulation costs no memory traffic per row), and loads the next row
// while it normalises the current one (two rows in flight per group). Mean and
// variance are two passes over the registers: warp shuffles within a row group of
// <= 32 threads, shared memory across the warps of a larger group.
#include <cuda_bf16.h>

#include <mutex>

#include "internal.h"
#include "ptx.cuh"

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

// Threads per block: several row groups of <= 32 threads, or one larger group.
template <int TPR>
constexpr int norm_block() {
  return TPR <= 32 ? kNormThreads : TPR;
}

template <int TPR>
__device__ __forceinline__ float group_sum(float v, float* red, int t) {
  constexpr int W = TPR < 32 ? TPR : 32;
#pragma unroll
  for (int o = W / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o, W);
  if constexpr (TPR > 32) {
    constexpr int NW = TPR / 32;
    if ((t & 31) == 0) red[t >> 5] = v;
    __syncthreads();
    v = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) v += red[w];
    __syncthreads();
  }
  return v;
}

template <int TPR>
__device__ __forceinline__ float group_max(float v, float* red, int t) {
  constexpr int W = TPR < 32 ? TPR : 32;
#pragma unroll
  for (int o = W / 2; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o, W));
  if constexpr (TPR > 32) {
    constexpr int NW = TPR / 32;
    if ((t & 31) == 0) red[t >> 5] = v;
    __syncthreads();
    v = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) v = fmaxf(v, red[w]);
    __syncthreads();
  }
  return v;
}

// OutT = uint8_t writes E4M3 codes of h / s with one scale per row, s = amax(|h|) / 448
// (1 for an all-zero row), into out and row_scale.
template <int TPR, int NU, bool MOD, typename OutT>
__global__ void __launch_bounds__(norm_block<TPR>()) layernorm_mod_kernel(
    const float* __restrict__ x, int64_t rows, int D, int L, const float* __restrict__ e,
    const float* __restrict__ mod_bias, int chunk, OutT* __restrict__ out, float eps,
    float* __restrict__ row_scale) {
  constexpr int G = norm_block<TPR>() / TPR;  // row groups per block
  __shared__ float red[TPR > 32 ? TPR / 32 : 1];
  const int group = threadIdx.x / TPR;
  const int t = threadIdx.x % TPR;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * G;
  const float inv_d = 1.0f / static_cast<float>(D);

  float shv[MOD ? NU : 1][8] = {};
  float scv[MOD ? NU : 1][8] = {};
  int64_t cur_b = -1;
  float va[NU][8], vb[NU][8];

  auto load = [&](float (&v)[NU][8], int64_t r) {
    const float* xr = x + (r < rows ? r : rows - 1) * D;
#pragma unroll
    for (int u = 0; u < NU; ++u) {
      const int col = (u * TPR + t) * 8;
      const float4 a = __ldcs(reinterpret_cast<const float4*>(xr + col));
      const float4 b = __ldcs(reinterpret_cast<const float4*>(xr + col + 4));
      v[u][0] = a.x; v[u][1] = a.y; v[u][2] = a.z; v[u][3] = a.w;
      v[u][4] = b.x; v[u][5] = b.y; v[u][6] = b.z; v[u][7] = b.w;
    }
  };
  auto process = [&](float (&v)[NU][8], int64_t r) {
    float s = 0.f;
#pragma unroll
    for (int u = 0; u < NU; ++u)
#pragma unroll
      for (int i = 0; i < 8; ++i) s += v[u][i];
    const float mean = group_sum<TPR>(s, red, t) * inv_d;
    float q = 0.f;
#pragma unroll
    for (int u = 0; u < NU; ++u)
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float c = v[u][i] - mean;
        q += c * c;
      }
    const float rstd = 1.0f / sqrtf(group_sum<TPR>(q, red, t) * inv_d + eps);
    if constexpr (sizeof(OutT) == 1) {
      // E4M3: the row's amax is a group reduction, taken by every group (also those past
      // the last row, which store nothing) so that the block's barriers stay uniform.
      if (MOD && r < rows) {
        const int64_t b = r / L;
        if (b != cur_b) {
          cur_b = b;
          const float* sh = e + (b * 6 + 3 * chunk) * D;
          const float* sc = sh + D;
          const float* bsh = mod_bias ? mod_bias + (3 * chunk) * D : nullptr;
#pragma unroll
          for (int u = 0; u < NU; ++u) {
            const int col = (u * TPR + t) * 8;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              shv[u][i] = sh[col + i] + (bsh ? bsh[col + i] : 0.f);
              scv[u][i] = 1.0f + sc[col + i] + (bsh ? bsh[D + col + i] : 0.f);
            }
          }
        }
      }
      float am = 0.f;
#pragma unroll
      for (int u = 0; u < NU; ++u)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          v[u][i] = (v[u][i] - mean) * rstd;
          if constexpr (MOD) v[u][i] = fmaf(v[u][i], scv[u][i], shv[u][i]);
          am = fmaxf(am, fabsf(v[u][i]));
        }
      am = group_max<TPR>(am, red, t);
      if (r >= rows) return;
      const float sc = am > 0.f ? __fdiv_rn(am, 448.0f) : 1.0f;
      if (t == 0) row_scale[r] = sc;
      uint8_t* orow = reinterpret_cast<uint8_t*>(out) + r * D;
#pragma unroll
      for (int u = 0; u < NU; ++u) {
        uint2 c;
        c.x = pack_e4m3x4(__fdiv_rn(v[u][0], sc), __fdiv_rn(v[u][1], sc), __fdiv_rn(v[u][2], sc),
                          __fdiv_rn(v[u][3], sc));
        c.y = pack_e4m3x4(__fdiv_rn(v[u][4], sc), __fdiv_rn(v[u][5], sc), __fdiv_rn(v[u][6], sc),
                          __fdiv_rn(v[u][7], sc));
        *reinterpret_cast<uint2*>(orow + (u * TPR + t) * 8) = c;
      }
    } else {
      if (r >= rows) return;
      if constexpr (MOD) {
        const int64_t b = r / L;
        if (b != cur_b) {
          cur_b = b;
          const float* sh = e + (b * 6 + 3 * chunk) * D;
          const float* sc = sh + D;
          const float* bsh = mod_bias ? mod_bias + (3 * chunk) * D : nullptr;
#pragma unroll
          for (int u = 0; u < NU; ++u) {
            const int col = (u * TPR + t) * 8;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              shv[u][i] = sh[col + i] + (bsh ? bsh[col + i] : 0.f);
              scv[u][i] = 1.0f + sc[col + i] + (bsh ? bsh[D + col + i] : 0.f);
            }
          }
        }
      }
      OutT* orow = out + r * D;
#pragma unroll
      for (int u = 0; u < NU; ++u) {
        float o[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          o[i] = (v[u][i] - mean) * rstd;
          if constexpr (MOD) o[i] = fmaf(o[i], scv[u][i], shv[u][i]);
        }
        store8<OutT>(orow + (u * TPR + t) * 8, o);
      }
    }
  };

  // The block's rows advance together (base is uniform across the block), so shuffles
  // and barriers never diverge; groups past the end load a valid row and skip stores.
  int64_t base = static_cast<int64_t>(blockIdx.x) * G;
  if (base >= rows) return;
  load(va, base + group);
  while (true) {
    const int64_t nb = base + stride;
    if (nb < rows) load(vb, nb + group);
    process(va, base + group);
    base = nb;
    if (base >= rows) break;
    const int64_t nb2 = base + stride;
    if (nb2 < rows) load(va, nb2 + group);
    process(vb, base + group);
    base = nb2;
    if (base >= rows) break;
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

int num_sms() {
  static int n[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  dev &= 63;
  if (n[dev] == 0) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    n[dev] = v > 0 ? v : 148;
  }
  return n[dev];
}

template <typename OutT, int TPR, int NU, bool MOD>
int launch_fixed(const float* x, int64_t rows, int D, int L, const float* e, const float* mb, int chunk,
                 OutT* out, float eps, cudaStream_t s, float* row_scale = nullptr) {
  constexpr int BT = norm_block<TPR>();
  constexpr int G = BT / TPR;
  auto kern = layernorm_mod_kernel<TPR, NU, MOD, OutT>;
  static int per_sm[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (per_sm[dev & 63] == 0) {
    int v = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, kern, BT, 0);
    per_sm[dev & 63] = v > 0 ? v : 1;
  }
  int64_t blocks = (rows + G - 1) / G;
  const int64_t cap = static_cast<int64_t>(per_sm[dev & 63]) * num_sms();
  if (blocks > cap) blocks = cap;
  kern<<<static_cast<unsigned>(blocks), BT, 0, s>>>(x, rows, D, L, e, mb, chunk, out, eps, row_scale);
  return check_launch();
}

template <typename OutT, bool MOD>
int launch_mod(const float* x, int64_t rows, int D, int L, const float* e, const float* mb, int chunk, OutT* out,
               float eps, cudaStream_t s) {
  const int units = D / 8;
#define WAN_LN_CASE(TPR, NU) \
  if (units == (TPR) * (NU)) return launch_fixed<OutT, TPR, NU, MOD>(x, rows, D, L, e, mb, chunk, out, eps, s);
  WAN_LN_CASE(8, 1)
  WAN_LN_CASE(16, 1)
  WAN_LN_CASE(32, 1)
  WAN_LN_CASE(32, 2)
  WAN_LN_CASE(64, 2)     // D = 1024
  WAN_LN_CASE(64, 3)     // D = 1536
  WAN_LN_CASE(64, 4)     // D = 2048
  WAN_LN_CASE(128, 3)    // D = 3072
  WAN_LN_CASE(128, 4)    // D = 4096
  WAN_LN_CASE(128, 5)    // D = 5120
#undef WAN_LN_CASE
  layernorm_mod_generic<OutT><<<static_cast<unsigned>(rows), kNormThreads, 0, s>>>(x, rows, D, L, e, mb, chunk,
                                                                                     out, eps);
  return check_launch();
}

template <typename OutT>
int launch_typed(const float* x, int64_t rows, int D, int L, const float* e, const float* mb, int chunk, OutT* out,
                 float eps, cudaStream_t s) {
  if (D % 8 != 0) {
    layernorm_mod_generic<OutT><<<static_cast<unsigned>(rows), kNormThreads, 0, s>>>(x, rows, D, L, e, mb, chunk,
                                                                                       out, eps);
    return check_launch();
  }
  return chunk >= 0 ? launch_mod<OutT, true>(x, rows, D, L, e, mb, chunk, out, eps, s)
                    : launch_mod<OutT, false>(x, rows, D, L, e, mb, chunk, out, eps, s);
}

template <bool MOD>
int launch_e4m3(const float* x, int64_t rows, int D, int L, const float* e, const float* mb, int chunk, uint8_t* out,
                float* row_scale, float eps, cudaStream_t s) {
  const int units = D / 8;
#define WAN_LN_CASE(TPR, NU)                                                                             \
  if (units == (TPR) * (NU))                                                                             \
    return launch_fixed<uint8_t, TPR, NU, MOD>(x, rows, D, L, e, mb, chunk, out, eps, s, row_scale);
  WAN_LN_CASE(32, 2)     // D = 512
  WAN_LN_CASE(64, 3)     // D = 1536
  WAN_LN_CASE(128, 5)    // D = 5120
#undef WAN_LN_CASE
  return WAN_ERR_UNSUPPORTED;
}

}  // namespace

int launch_layernorm_e4m3(const float* x, int64_t rows, int D, int L, const float* e, const float* mod_bias,
                          int chunk, void* out, float* row_scale, float eps, cudaStream_t s) {
  if (rows == 0) return WAN_OK;
  if (D % 8 != 0) return WAN_ERR_UNSUPPORTED;
  trace_launch_begin(WAN_KIND_NORM, s, static_cast<double>(rows) * (D * 5.0 + 4.0));
  const int st = chunk >= 0 ? launch_e4m3<true>(x, rows, D, L, e, mod_bias, chunk, static_cast<uint8_t*>(out),
                                                row_scale, eps, s)
                            : launch_e4m3<false>(x, rows, D, L, e, mod_bias, chunk, static_cast<uint8_t*>(out),
                                                 row_scale, eps, s);
  trace_launch_end(WAN_KIND_NORM, s);
  return st;
}

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
