// fp32 path of the library (wan_dit_config.dtype == WAN_F32): CUDA-core GEMM and
// attention kernels with full fp32 arithmetic, for workloads whose tolerance rules out
// reduced-precision tensor-core inputs. Same semantics and epilogues as the bf16
// tensor-core kernels in gemm_tc.cu and attn_tc.cu.
#include <math.h>

#include "internal.h"

namespace wan {
namespace {

constexpr int kT = 64;   // output tile
constexpr int kKT = 16;  // reduction tile

__device__ __forceinline__ float gelu_tanh_exact(float v) {
  return 0.5f * v * (1.0f + tanhf(0.7978845608028654f * (v + 0.044715f * v * v * v)));
}

__global__ void __launch_bounds__(256) gemm_f32_kernel(const float* __restrict__ A, int64_t lda,
                                                       const float* __restrict__ W, int kw,
                                                       const float* __restrict__ bias, void* out, int M, int N,
                                                       int K, GemmEpi epi) {
  __shared__ float sa[kKT][kT + 1];
  __shared__ float sw[kKT][kT + 1];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int m0 = blockIdx.y * kT, n0 = blockIdx.x * kT;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += kKT) {
    for (int i = threadIdx.x; i < kT * kKT; i += 256) {
      const int r = i / kKT, c = i % kKT;
      const int m = m0 + r, n = n0 + r, k = k0 + c;
      sa[c][r] = (m < M && k < K) ? A[static_cast<int64_t>(m) * lda + k] : 0.f;
      sw[c][r] = (n < N && k < K) ? W[static_cast<int64_t>(n) * kw + (k % kw)] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c < kKT; ++c) {
      float a[4], w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = sa[c][ty * 4 + i];
        w[i] = sw[c][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], w[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= N) continue;
      float v = acc[i][j] + (bias ? bias[n] : 0.f);
      if (epi.kind == WAN_EPI_STORE || epi.kind == WAN_EPI_F32) {
        static_cast<float*>(out)[static_cast<int64_t>(m) * epi.ldo + n] = v;
      } else if (epi.kind == WAN_EPI_GELU) {
        static_cast<float*>(out)[static_cast<int64_t>(m) * epi.ldo + n] = gelu_tanh_exact(v);
      } else if (epi.kind == WAN_EPI_RESIDUAL) {
        float g = 1.f;
        if (epi.gate) {
          g = epi.gate[static_cast<int64_t>(m / epi.rows_per_batch) * epi.gate_bstride + n];
          if (epi.gate_bias) g += epi.gate_bias[n];
        }
        static_cast<float*>(out)[static_cast<int64_t>(m) * epi.ldo + n] += g * v;
      } else {  // head scatter
        const int L = epi.rows_per_batch;
        const int b = m / L, l = m % L;
        const int Hh = epi.sc_H / 2, Wh = epi.sc_W / 2;
        const int f = l / (Hh * Wh), ii = (l / Wh) % Hh, jj = l % Wh;
        const int c = n >> 2, ph = (n >> 1) & 1, pw = n & 1;
        const int64_t idx = ((static_cast<int64_t>(b) * epi.sc_C + c) * epi.sc_F + f) * epi.sc_H * epi.sc_W +
                            static_cast<int64_t>(2 * ii + ph) * epi.sc_W + (2 * jj + pw);
        static_cast<float*>(out)[idx] = v;
      }
    }
  }
}

constexpr int kAttnSimtThreads = 128;

// One block per (query row, head, sample): scores in shared memory, exact softmax.
__global__ void __launch_bounds__(kAttnSimtThreads) attn_f32_kernel(
    const float* __restrict__ q, int64_t qs, int qc, const float* __restrict__ k, int64_t ks, int kc,
    const float* __restrict__ v, int64_t vs, int vc, float* __restrict__ o, int64_t os, int oc, int Lq, int Lk,
    int d, float scale) {
  extern __shared__ float sm[];
  float* sq = sm;        // [d]
  float* sc = sm + 128;  // [Lk]
  __shared__ float red[kAttnSimtThreads / 32];
  const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const float* qr = q + (static_cast<int64_t>(b) * Lq + i) * qs + qc + h * d;
  for (int c = threadIdx.x; c < d; c += kAttnSimtThreads) sq[c] = qr[c];
  __syncthreads();
  const float* kb = k + static_cast<int64_t>(b) * Lk * ks + kc + h * d;
  const float* vb = v + static_cast<int64_t>(b) * Lk * vs + vc + h * d;
  float mx = -INFINITY;
  for (int j = threadIdx.x; j < Lk; j += kAttnSimtThreads) {
    const float* kr = kb + static_cast<int64_t>(j) * ks;
    float s = 0.f;
    for (int c = 0; c < d; ++c) s = fmaf(sq[c], kr[c], s);
    s *= scale;
    sc[j] = s;
    mx = fmaxf(mx, s);
  }
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  mx = red[0];
  for (int w = 1; w < kAttnSimtThreads / 32; ++w) mx = fmaxf(mx, red[w]);
  __syncthreads();
  float sum = 0.f;
  for (int j = threadIdx.x; j < Lk; j += kAttnSimtThreads) {
    const float pj = expf(sc[j] - mx);
    sc[j] = pj;
    sum += pj;
  }
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = sum;
  __syncthreads();
  sum = 0.f;
  for (int w = 0; w < kAttnSimtThreads / 32; ++w) sum += red[w];
  float* orow = o + (static_cast<int64_t>(b) * Lq + i) * os + oc + h * d;
  for (int c = threadIdx.x; c < d; c += kAttnSimtThreads) {
    float acc = 0.f;
    for (int j = 0; j < Lk; ++j) acc = fmaf(sc[j], vb[static_cast<int64_t>(j) * vs + c], acc);
    orow[c] = acc / sum;
  }
}

}  // namespace

int launch_gemm_simt(const float* A, int64_t lda, const float* W, const float* bias, void* out, int M, int N, int K,
                     int w_k_period, const GemmEpi& epi, cudaStream_t s) {
  if (M == 0 || N == 0) return WAN_OK;
  const int kw = w_k_period > 0 ? w_k_period : K;
  dim3 grid((N + kT - 1) / kT, (M + kT - 1) / kT);
  trace_launch_begin(WAN_KIND_GEMM, s, 2.0 * M * N * K);
  gemm_f32_kernel<<<grid, 256, 0, s>>>(A, lda, W, kw, bias, out, M, N, K, epi);
  int st = check_launch();
  trace_launch_end(WAN_KIND_GEMM, s);
  return st;
}

int launch_attn_simt(AttnOperand q, AttnOperand k, AttnOperand v, void* o, int64_t o_row_stride, int o_col0, int B,
                     int H, int Lq, int Lk, int d, cudaStream_t s) {
  if (B == 0 || Lq == 0) return WAN_OK;
  if (Lk <= 0 || Lk > 8192 || d > 128) return WAN_ERR_SHAPE;
  dim3 grid(Lq, H, B);
  const size_t smem = (128 + static_cast<size_t>(Lk)) * sizeof(float);
  trace_launch_begin(WAN_KIND_ATTN, s, 4.0 * B * H * static_cast<double>(Lq) * Lk * d);
  attn_f32_kernel<<<grid, kAttnSimtThreads, smem, s>>>(
      static_cast<const float*>(q.ptr), q.row_stride, q.col0, static_cast<const float*>(k.ptr), k.row_stride,
      k.col0, static_cast<const float*>(v.ptr), v.row_stride, v.col0, static_cast<float*>(o), o_row_stride,
      o_col0, Lq, Lk, d, static_cast<float>(1.0 / sqrt(static_cast<double>(d))));
  int st = check_launch();
  trace_launch_end(WAN_KIND_ATTN, s);
  return st;
}

}  // namespace wan
