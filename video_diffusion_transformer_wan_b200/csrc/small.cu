// Small kernels of the Wan 2.1 DiT forward path ("Wan: Open and Advanced Large-Scale
// Video Generative Models", sections "Diffusion Transformer", "I2V 架构扩展" and
// "训练方法"): the (1,2,2) patch gather feeding the patchify GEMM, the shared timestep
// MLP, I2V input fusion, and the rectified-flow interpolation and loss.
#include <cuda_bf16.h>
#include <math.h>

#include "internal.h"
#include "ptx.cuh"

namespace wan {
namespace {

template <typename T>
__device__ __forceinline__ float ld(const T* p, int64_t i);
template <>
__device__ __forceinline__ float ld<float>(const float* p, int64_t i) {
  return p[i];
}
template <>
__device__ __forceinline__ float ld<__nv_bfloat16>(const __nv_bfloat16* p, int64_t i) {
  return __bfloat162float(p[i]);
}
template <typename T>
__device__ __forceinline__ T cvt(float v);
template <>
__device__ __forceinline__ float cvt<float>(float v) {
  return v;
}
template <>
__device__ __forceinline__ __nv_bfloat16 cvt<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// patches[b*L + (f*Hh + i)*Wh + j, c*4 + ph*2 + pw] = latent[b, c, f, 2i+ph, 2j+pw]
// One thread per (token, channel): two 2-element reads, one 4-element write.
template <typename T>
__global__ void patch_gather_kernel(const T* __restrict__ lat, int B, int C, int F, int H, int W,
                                    T* __restrict__ out) {
  const int Hh = H / 2, Wh = W / 2;
  const int64_t L = static_cast<int64_t>(F) * Hh * Wh;
  const int64_t total = static_cast<int64_t>(B) * L * C;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(idx % C);
    const int64_t tok = idx / C;
    const int b = static_cast<int>(tok / L);
    const int64_t l = tok % L;
    const int f = static_cast<int>(l / (Hh * Wh));
    const int i = static_cast<int>((l / Wh) % Hh);
    const int j = static_cast<int>(l % Wh);
    const T* src = lat + ((static_cast<int64_t>(b) * C + c) * F + f) * H * W + static_cast<int64_t>(2 * i) * W + 2 * j;
    T* dst = out + tok * (C * 4) + c * 4;
    dst[0] = src[0];
    dst[1] = src[1];
    dst[2] = src[W];
    dst[3] = src[W + 1];
  }
}

constexpr int kTimeThreads = 512;
constexpr int kTimeOutPerBlock = 256;
constexpr int kTimeRows = 4;  // weight rows a warp reduces at once (independent loads in flight)

// 16-byte vector loads of weight rows, widened to fp32.
template <typename T>
struct Vec16;
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void load(const __nv_bfloat16* p, float (&f)[8]) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 v = __bfloat1622float2(h[i]);
      f[2 * i] = v.x;
      f[2 * i + 1] = v.y;
    }
  }
};
template <>
struct Vec16<float> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void load(const float* p, float (&f)[4]) {
    const float4 u = __ldg(reinterpret_cast<const float4*>(p));
    f[0] = u.x; f[1] = u.y; f[2] = u.z; f[3] = u.w;
  }
};

// acc[r] = sum_k w[(row0 + r) * n + k] * v[k] for kTimeRows rows (rows >= nrows are
// computed on a valid row and ignored by the caller); the result is in every lane.
template <typename T>
__device__ __forceinline__ void warp_dot_rows(const T* __restrict__ w, int row0, int nrows, int n,
                                              const float* __restrict__ v, int lane, float (&acc)[kTimeRows]) {
  constexpr int V = Vec16<T>::N;
  const T* rp[kTimeRows];
#pragma unroll
  for (int r = 0; r < kTimeRows; ++r) {
    acc[r] = 0.f;
    rp[r] = w + static_cast<int64_t>(min(row0 + r, nrows - 1)) * n;
  }
  const int nv = (n / V) * V;
  for (int k = lane * V; k < nv; k += 32 * V) {
    float f[kTimeRows][V];
#pragma unroll
    for (int r = 0; r < kTimeRows; ++r) Vec16<T>::load(rp[r] + k, f[r]);
#pragma unroll
    for (int r = 0; r < kTimeRows; ++r)
#pragma unroll
      for (int i = 0; i < V; ++i) acc[r] = fmaf(f[r][i], v[k + i], acc[r]);
  }
  for (int k = nv + lane; k < n; k += 32)
#pragma unroll
    for (int r = 0; r < kTimeRows; ++r) acc[r] = fmaf(ld(rp[r], k), v[k], acc[r]);
#pragma unroll
  for (int r = 0; r < kTimeRows; ++r)
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], off);
}

// e[b, m] = sum_n w2[m, n] silu(sum_k w1[n, k] emb_k(t_b) + b1[n]) + b2[m], m < 6D.
// Each block recomputes the sinusoid (double-precision arguments) and the D hidden
// units in shared memory (W1 is small and L2-resident), then produces 256 outputs;
// a warp reduces kTimeRows weight rows at a time with 16-byte loads.
template <typename T>
__global__ void __launch_bounds__(kTimeThreads) time_mlp_kernel(const float* __restrict__ t, int D, int freq_dim,
                                                                 const T* __restrict__ w1, const T* __restrict__ b1,
                                                                 const T* __restrict__ w2, const T* __restrict__ b2,
                                                                 float* __restrict__ e) {
  extern __shared__ float sm[];
  float* emb = sm;              // [freq_dim]
  float* hid = sm + freq_dim;   // [D]
  const int b = blockIdx.y;
  const int half = freq_dim / 2;
  const double tb = static_cast<double>(t[b]);
  for (int k = threadIdx.x; k < half; k += kTimeThreads) {
    const double f = pow(10000.0, -static_cast<double>(k) / half);
    emb[k] = static_cast<float>(cos(tb * f));
    emb[half + k] = static_cast<float>(sin(tb * f));
  }
  __syncthreads();
  constexpr int kWarps = kTimeThreads / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int n0 = warp * kTimeRows; n0 < D; n0 += kWarps * kTimeRows) {
    float acc[kTimeRows];
    warp_dot_rows(w1, n0, D, freq_dim, emb, lane, acc);
    if (lane < kTimeRows && n0 + lane < D) {
      float a = acc[0];
#pragma unroll
      for (int r = 1; r < kTimeRows; ++r)
        if (lane == r) a = acc[r];
      const float z = a + ld(b1, n0 + lane);
      hid[n0 + lane] = z / (1.0f + expf(-z));
    }
  }
  __syncthreads();
  const int m_beg = blockIdx.x * kTimeOutPerBlock;
  const int m_end = min(6 * D, m_beg + kTimeOutPerBlock);
  for (int m0 = m_beg + warp * kTimeRows; m0 < m_end; m0 += kWarps * kTimeRows) {
    float acc[kTimeRows];
    warp_dot_rows(w2, m0, 6 * D, D, hid, lane, acc);
    if (lane < kTimeRows && m0 + lane < m_end) {
      float a = acc[0];
#pragma unroll
      for (int r = 1; r < kTimeRows; ++r)
        if (lane == r) a = acc[r];
      e[static_cast<int64_t>(b) * 6 * D + m0 + lane] = a + ld(b2, m0 + lane);
    }
  }
}

// The same MLP in two launches when a scratch for the hidden units is available, so
// that neither layer is recomputed per block and both spread over many SMs:
// time_hidden_kernel writes hid[b, n] (kTimeSplitRows units per block),
// time_out_kernel reads hid[b] into shared memory and writes kTimeSplitRows outputs.
constexpr int kTimeSplitThreads = 256;
constexpr int kTimeSplitRows = 64;

template <typename T>
__global__ void __launch_bounds__(kTimeSplitThreads) time_hidden_kernel(const float* __restrict__ t, int D,
                                                                        int freq_dim, const T* __restrict__ w1,
                                                                        const T* __restrict__ b1,
                                                                        float* __restrict__ hid) {
  extern __shared__ float emb[];  // [freq_dim]
  const int b = blockIdx.y;
  const int half = freq_dim / 2;
  const double tb = static_cast<double>(t[b]);
  for (int k = threadIdx.x; k < half; k += kTimeSplitThreads) {
    const double f = pow(10000.0, -static_cast<double>(k) / half);
    emb[k] = static_cast<float>(cos(tb * f));
    emb[half + k] = static_cast<float>(sin(tb * f));
  }
  __syncthreads();
  constexpr int kWarps = kTimeSplitThreads / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_end = min(D, (blockIdx.x + 1) * kTimeSplitRows);
  for (int n0 = blockIdx.x * kTimeSplitRows + warp * kTimeRows; n0 < n_end; n0 += kWarps * kTimeRows) {
    float acc[kTimeRows];
    warp_dot_rows(w1, n0, D, freq_dim, emb, lane, acc);
    if (lane < kTimeRows && n0 + lane < n_end) {
      float a = acc[0];
#pragma unroll
      for (int r = 1; r < kTimeRows; ++r)
        if (lane == r) a = acc[r];
      const float z = a + ld(b1, n0 + lane);
      hid[static_cast<int64_t>(b) * D + n0 + lane] = z / (1.0f + expf(-z));
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kTimeSplitThreads) time_out_kernel(const float* __restrict__ hid, int D,
                                                                     const T* __restrict__ w2,
                                                                     const T* __restrict__ b2,
                                                                     float* __restrict__ e) {
  extern __shared__ float h[];  // [D]
  const int b = blockIdx.y;
  for (int n = threadIdx.x; n < D; n += kTimeSplitThreads) h[n] = hid[static_cast<int64_t>(b) * D + n];
  __syncthreads();
  constexpr int kWarps = kTimeSplitThreads / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_end = min(6 * D, (blockIdx.x + 1) * kTimeSplitRows);
  for (int m0 = blockIdx.x * kTimeSplitRows + warp * kTimeRows; m0 < m_end; m0 += kWarps * kTimeRows) {
    float acc[kTimeRows];
    warp_dot_rows(w2, m0, 6 * D, D, h, lane, acc);
    if (lane < kTimeRows && m0 + lane < m_end) {
      float a = acc[0];
#pragma unroll
      for (int r = 1; r < kTimeRows; ++r)
        if (lane == r) a = acc[r];
      e[static_cast<int64_t>(b) * 6 * D + m0 + lane] = a + ld(b2, m0 + lane);
    }
  }
}

// out[b, c, f, y, x]: c < 16 noise, c < 32 condition latent, c < 36 the frame mask,
// where latent frame f, mask channel mc takes pixel frame 0 for f == 0 (the first frame
// repeated 4 times) and pixel frame 4f + mc - 3 otherwise.
template <typename T>
__global__ void i2v_input_kernel(const T* __restrict__ noise, const T* __restrict__ cond,
                                 const uint8_t* __restrict__ keep, int B, int F, int H, int W, T* __restrict__ out) {
  const int64_t plane = static_cast<int64_t>(F) * H * W;
  const int64_t total = static_cast<int64_t>(B) * 36 * plane;
  const int nkeep = 1 + 4 * (F - 1);
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t within = idx % plane;
    const int c = static_cast<int>((idx / plane) % 36);
    const int b = static_cast<int>(idx / (36 * plane));
    T v;
    if (c < 16) {
      v = noise[(static_cast<int64_t>(b) * 16 + c) * plane + within];
    } else if (c < 32) {
      v = cond[(static_cast<int64_t>(b) * 16 + (c - 16)) * plane + within];
    } else {
      const int f = static_cast<int>(within / (static_cast<int64_t>(H) * W));
      const int mc = c - 32;
      const int frame = f == 0 ? 0 : 4 * f + mc - 3;
      v = cvt<T>(keep[static_cast<int64_t>(b) * nkeep + frame] ? 1.0f : 0.0f);
    }
    out[idx] = v;
  }
}

template <typename T>
__global__ void flow_input_kernel(const T* __restrict__ x1, const T* __restrict__ x0, const float* __restrict__ u,
                                  int B, int64_t n, T* __restrict__ xt, float* __restrict__ t_out) {
  const int64_t total = static_cast<int64_t>(B) * n;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float ub = u[idx / n];
    xt[idx] = cvt<T>(ub * ld(x1, idx) + (1.0f - ub) * ld(x0, idx));
    if (t_out && idx % n == 0) t_out[idx / n] = 1000.0f * ub;
  }
}

// One block per sample: loss[b] = mean((v - (x1 - x0))^2), accumulated in double in a
// fixed order (deterministic).
template <typename T>
__global__ void __launch_bounds__(256) flow_loss_kernel(const float* __restrict__ v, const T* __restrict__ x1,
                                                        const T* __restrict__ x0, int64_t n, float* __restrict__ loss) {
  __shared__ double red[8];
  const int b = blockIdx.x;
  const int64_t base = static_cast<int64_t>(b) * n;
  double acc = 0.0;
  for (int64_t i = threadIdx.x; i < n; i += 256) {
    const double d = static_cast<double>(v[base + i]) - (static_cast<double>(ld(x1, base + i)) - ld(x0, base + i));
    acc += d * d;
  }
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int w = 0; w < 8; ++w) s += red[w];
    loss[b] = static_cast<float>(s / static_cast<double>(n));
  }
}

// Sampler set-up: the 2B-sample DiT input (both halves = the caller's input, which
// holds the noise in its first n elements per sample and, for I2V, fixed condition
// channels after them), the fp32 state x = noise, and the timestep of step 0.
template <typename T>
__global__ void sampler_init_kernel(const T* __restrict__ input, int B, int64_t n, int64_t in_stride,
                                    float* __restrict__ x, T* __restrict__ in2, float* __restrict__ t) {
  const int64_t total = static_cast<int64_t>(B) * in_stride;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t b = idx / in_stride, i = idx % in_stride;
    const T v = input[idx];
    in2[idx] = v;
    in2[static_cast<int64_t>(B) * in_stride + idx] = v;
    if (i < n) x[b * n + i] = ld(input, idx);
    if (idx < 2 * B) t[idx] = 0.0f;
  }
}

// One guided Euler step. Both passes ran (skip = 0): v = [v_c (B samples) | v_u (B
// samples)], delta = v_c - v_u (kept in `delta` when it is not null) and
// x += dt * (v_u + g delta). The unconditional pass was skipped (skip = 1): v = v_c
// (B samples) and x += dt * (v_c + (g - 1) delta) with the kept delta. The new x
// (rounded to the activation type) goes into the first n elements of both halves of
// the next DiT input, and the timestep becomes t_next.
template <typename T>
__global__ void euler_cfg_kernel(const float* __restrict__ v, int B, int64_t n, int64_t in_stride, float dt,
                                 float g, float* __restrict__ x, T* __restrict__ in2, float* __restrict__ t,
                                 float t_next, float* __restrict__ delta, int skip) {
  const int64_t total = static_cast<int64_t>(B) * n;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t b = idx / n, i = idx % n;
    const float vc = v[idx];
    float vel;
    if (skip) {
      vel = vc + (g - 1.0f) * delta[idx];
    } else {
      const float vu = v[total + idx];
      const float d = vc - vu;
      if (delta) delta[idx] = d;
      vel = vu + g * d;
    }
    const float xv = x[idx] + dt * vel;
    x[idx] = xv;
    const T xt = cvt<T>(xv);
    in2[b * in_stride + i] = xt;
    in2[(b + B) * in_stride + i] = xt;
    if (idx < 2 * B) t[idx] = t_next;
  }
}

// One thread waits on a barrier that nothing arrives at: the bounded wait gives up
// after its limit and records the timeout in the device error flag.
__global__ void wait_timeout_probe_kernel(int* err) {
  __shared__ uint64_t bar;
  mbar_init(&bar, 1);
  fence_mbar_init();
  mbar_wait(&bar, 0, err);
}

unsigned grid_for(int64_t total, int threads) {
  int64_t g = (total + threads - 1) / threads;
  if (g > 148 * 64) g = 148 * 64;
  return static_cast<unsigned>(g < 1 ? 1 : g);
}

}  // namespace

int launch_sampler_init(const void* input, int B, int64_t n, int64_t in_stride, float* x, void* in2, float* t,
                        int dtype, cudaStream_t s) {
  const int64_t total = static_cast<int64_t>(B) * in_stride;
  if (total == 0) return WAN_OK;
  trace_launch_begin(WAN_KIND_SMALL, s, static_cast<double>(total) * dtype_size(dtype) * 3.0);
  if (dtype == WAN_BF16)
    sampler_init_kernel<__nv_bfloat16><<<grid_for(total, 256), 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(input), B, n, in_stride, x, static_cast<__nv_bfloat16*>(in2), t);
  else
    sampler_init_kernel<float><<<grid_for(total, 256), 256, 0, s>>>(static_cast<const float*>(input), B, n,
                                                                    in_stride, x, static_cast<float*>(in2), t);
  int st = check_launch();
  trace_launch_end(WAN_KIND_SMALL, s);
  return st;
}

int launch_euler_cfg(const float* v, int B, int64_t n, int64_t in_stride, float dt, float g, float* x, void* in2,
                     float* t, float t_next, int dtype, cudaStream_t s, float* delta, bool skip) {
  const int64_t total = static_cast<int64_t>(B) * n;
  if (total == 0) return WAN_OK;
  trace_launch_begin(WAN_KIND_SMALL, s, static_cast<double>(total) * (16.0 + 2.0 * dtype_size(dtype)));
  if (dtype == WAN_BF16)
    euler_cfg_kernel<__nv_bfloat16><<<grid_for(total, 256), 256, 0, s>>>(
        v, B, n, in_stride, dt, g, x, static_cast<__nv_bfloat16*>(in2), t, t_next, delta, skip ? 1 : 0);
  else
    euler_cfg_kernel<float><<<grid_for(total, 256), 256, 0, s>>>(
        v, B, n, in_stride, dt, g, x, static_cast<float*>(in2), t, t_next, delta, skip ? 1 : 0);
  int st = check_launch();
  trace_launch_end(WAN_KIND_SMALL, s);
  return st;
}

int launch_patch_gather(const void* latent, int B, int C, int F, int H, int W, void* patches, int dtype,
                        cudaStream_t s) {
  const int64_t total = static_cast<int64_t>(B) * F * (H / 2) * (W / 2) * C;
  if (total == 0) return WAN_OK;
  trace_launch_begin(WAN_KIND_SMALL, s);
  if (dtype == WAN_BF16)
    patch_gather_kernel<__nv_bfloat16><<<grid_for(total, 256), 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(latent), B, C, F, H, W, static_cast<__nv_bfloat16*>(patches));
  else
    patch_gather_kernel<float><<<grid_for(total, 256), 256, 0, s>>>(static_cast<const float*>(latent), B, C, F, H,
                                                                    W, static_cast<float*>(patches));
  int st = check_launch();
  trace_launch_end(WAN_KIND_SMALL, s);
  return st;
}

int launch_time_mlp(const float* t, int B, int D, int freq_dim, const void* w1, const void* b1, const void* w2,
                    const void* b2, float* e_out, int dtype, cudaStream_t s, float* hid_scratch) {
  if (B == 0) return WAN_OK;
  if (hid_scratch) {
    if (static_cast<size_t>(D) * sizeof(float) > 48 * 1024) return WAN_ERR_SHAPE;
    trace_launch_begin(WAN_KIND_SMALL, s);
    const dim3 g1((D + kTimeSplitRows - 1) / kTimeSplitRows, B), g2((6 * D + kTimeSplitRows - 1) / kTimeSplitRows, B);
    const size_t sm1 = static_cast<size_t>(freq_dim) * sizeof(float), sm2 = static_cast<size_t>(D) * sizeof(float);
    if (dtype == WAN_BF16) {
      time_hidden_kernel<__nv_bfloat16><<<g1, kTimeSplitThreads, sm1, s>>>(
          t, D, freq_dim, static_cast<const __nv_bfloat16*>(w1), static_cast<const __nv_bfloat16*>(b1), hid_scratch);
      time_out_kernel<__nv_bfloat16><<<g2, kTimeSplitThreads, sm2, s>>>(
          hid_scratch, D, static_cast<const __nv_bfloat16*>(w2), static_cast<const __nv_bfloat16*>(b2), e_out);
    } else {
      time_hidden_kernel<float><<<g1, kTimeSplitThreads, sm1, s>>>(
          t, D, freq_dim, static_cast<const float*>(w1), static_cast<const float*>(b1), hid_scratch);
      time_out_kernel<float><<<g2, kTimeSplitThreads, sm2, s>>>(
          hid_scratch, D, static_cast<const float*>(w2), static_cast<const float*>(b2), e_out);
    }
    count_launches(1);  // two kernels in this bracket
    const int st = check_launch();
    trace_launch_end(WAN_KIND_SMALL, s);
    return st;
  }
  dim3 grid((6 * D + kTimeOutPerBlock - 1) / kTimeOutPerBlock, B);
  const size_t smem = static_cast<size_t>(freq_dim + D) * sizeof(float);
  if (smem > 48 * 1024) return WAN_ERR_SHAPE;
  trace_launch_begin(WAN_KIND_SMALL, s);
  if (dtype == WAN_BF16)
    time_mlp_kernel<__nv_bfloat16><<<grid, kTimeThreads, smem, s>>>(
        t, D, freq_dim, static_cast<const __nv_bfloat16*>(w1), static_cast<const __nv_bfloat16*>(b1),
        static_cast<const __nv_bfloat16*>(w2), static_cast<const __nv_bfloat16*>(b2), e_out);
  else
    time_mlp_kernel<float><<<grid, kTimeThreads, smem, s>>>(t, D, freq_dim, static_cast<const float*>(w1),
                                                           static_cast<const float*>(b1),
                                                           static_cast<const float*>(w2),
                                                           static_cast<const float*>(b2), e_out);
  int st = check_launch();
  trace_launch_end(WAN_KIND_SMALL, s);
  return st;
}

int launch_i2v_input(const void* noise, const void* cond, const uint8_t* keep, int B, int F, int H, int W, void* out,
                     int dtype, cudaStream_t s) {
  const int64_t total = static_cast<int64_t>(B) * 36 * F * H * W;
  if (total == 0) return WAN_OK;
  trace_launch_begin(WAN_KIND_SMALL, s);
  if (dtype == WAN_BF16)
    i2v_input_kernel<__nv_bfloat16><<<grid_for(total, 256), 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(noise), static_cast<const __nv_bfloat16*>(cond), keep, B, F, H, W,
        static_cast<__nv_bfloat16*>(out));
  else
    i2v_input_kernel<float><<<grid_for(total, 256), 256, 0, s>>>(static_cast<const float*>(noise),
                                                                 static_cast<const float*>(cond), keep, B, F, H, W,
                                                                 static_cast<float*>(out));
  int st = check_launch();
  trace_launch_end(WAN_KIND_SMALL, s);
  return st;
}

int launch_flow_input(const void* x1, const void* x0, const float* u, int B, int64_t n, void* xt, float* t_out,
                      int dtype, cudaStream_t s) {
  const int64_t total = static_cast<int64_t>(B) * n;
  if (total == 0) return WAN_OK;
  trace_launch_begin(WAN_KIND_SMALL, s);
  if (dtype == WAN_BF16)
    flow_input_kernel<__nv_bfloat16><<<grid_for(total, 256), 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(x1), static_cast<const __nv_bfloat16*>(x0), u, B, n,
        static_cast<__nv_bfloat16*>(xt), t_out);
  else
    flow_input_kernel<float><<<grid_for(total, 256), 256, 0, s>>>(static_cast<const float*>(x1),
                                                                  static_cast<const float*>(x0), u, B, n,
                                                                  static_cast<float*>(xt), t_out);
  int st = check_launch();
  trace_launch_end(WAN_KIND_SMALL, s);
  return st;
}

int launch_flow_loss(const float* v, const void* x1, const void* x0, int B, int64_t n, float* loss, int dtype,
                     cudaStream_t s) {
  if (B == 0) return WAN_OK;
  trace_launch_begin(WAN_KIND_SMALL, s);
  if (dtype == WAN_BF16)
    flow_loss_kernel<__nv_bfloat16><<<B, 256, 0, s>>>(v, static_cast<const __nv_bfloat16*>(x1),
                                                      static_cast<const __nv_bfloat16*>(x0), n, loss);
  else
    flow_loss_kernel<float><<<B, 256, 0, s>>>(v, static_cast<const float*>(x1), static_cast<const float*>(x0), n,
                                              loss);
  int st = check_launch();
  trace_launch_end(WAN_KIND_SMALL, s);
  return st;
}

int launch_wait_timeout_probe(cudaStream_t s) {
  wait_timeout_probe_kernel<<<1, 1, 0, s>>>(device_error_flag());
  count_launches(1);
  return check_launch();
}

}  // namespace wan
