// Kernel (b): flash-attention forward on the sm_100a tensor cores for the Wan 2.1 DiT
// ("Wan: Open and Advanced Large-Scale Video Generative Models", section "Diffusion
// Transformer": full spatio-temporal self-attention over all L video tokens, and text
// cross-attention over 512 umT5 tokens in every block). softmax(q k^T / sqrt(d)) v per
// head, non-causal, bf16 inputs, fp32 accumulation and fp32 softmax, head_dim 128.
//
// One CTA = one 128-row query tile of one (sample, head); 192 threads:
//   warp 0   : TMA producer - Q once, then K_0, V_0, K_1, V_1, ... through a 4-stage
//              ring of 32 KB tiles (128 rows x 128 dims, two 64-dim halves with
//              128-byte swizzle);
//   warp 1   : one thread issues tcgen05.mma: S_j = Q K_j^T into one of two TMEM S
//              buffers (so QK^T of tile j+1 runs while tile j is in softmax), then
//              O += P_{j-1} V_{j-1} into the TMEM O accumulator (V is an MN-major
//              operand, no transpose pass);
//   warps 2-5: softmax, one thread per query row: tcgen05.ld of its S row, masking of
//              the ragged last key tile, running max and sum in fp32, exponentials
//              with ex2, P rounded to bf16 into swizzled shared memory for the PV MMA.
//              The running max used as the exponent base is only moved when the new
//              row max exceeds it by more than 2^8 in probability terms; O (in TMEM)
//              and the sum are rescaled then. Softmax is invariant to the base, and
//              p <= 256 stays well inside fp32 and bf16 range, so the result is the
//              same softmax. At the end O is divided by the sum and stored as bf16.
#include <cuda_bf16.h>

#include <math.h>

#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace wan {
namespace {

constexpr int kAttnThreads = 192;
constexpr int kTile = 128;            // query rows per CTA = key rows per tile
constexpr int kHd = 128;              // head dim
constexpr int kStages = 4;            // K/V ring depth
constexpr int kTileBytes = kTile * kHd * 2;   // 32 KB
constexpr int kHalfBytes = kTileBytes / 2;    // one 64-column half
constexpr size_t kAttnSmem = 1024 + static_cast<size_t>(kTileBytes) * (1 + kStages + 2) + 256;
constexpr float kRescaleLog2 = 8.0f;  // move the exponent base when the max grows by > 2^8

struct AttnParams {
  int Lq, Lk, H;
  int q_col0, k_col0, v_col0;
  float scale_log2;       // log2(e) / sqrt(d)
  __nv_bfloat16* o;
  int64_t o_row_stride;
  int64_t o_batch_stride;
  int o_col0;
  int* err;
};

__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                       const __grid_constant__ CUtensorMap mapV, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = sQ + kTileBytes;
  uint8_t* sP = sKV + kStages * kTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + 2 * kTileBytes);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + kStages;
  uint64_t* s_full = kv_empty + kStages;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;
  uint64_t* o_done = p_full + 2;
  uint64_t* drain = o_done + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int q0 = blockIdx.x * kTile;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int nkv = (p.Lk + kTile - 1) / kTile;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 128);
      mbar_init(&p_full[i], 128);
      mbar_init(&o_done[i], 1);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mapQ);
    tma_prefetch_desc(&mapK);
    tma_prefetch_desc(&mapV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const uint32_t tmem_o = tmem_base + 256;

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, kTileBytes);
      const int qc = p.q_col0 + h * kHd;
      tma_load_3d(sQ, &mapQ, q_full, qc, q0, b);
      tma_load_3d(sQ + kHalfBytes, &mapQ, q_full, qc + 64, q0, b);
      const int n_loads = 2 * nkv;
      int issued = 0;
      for (int ld = 0; ld < n_loads; ++ld) {
        const int stage = ld % kStages;
        const uint32_t phase = static_cast<uint32_t>((ld / kStages) & 1);
        if (!mbar_wait(&kv_empty[stage], phase ^ 1u, p.err)) break;
        const bool is_v = ld & 1;
        const int j = ld >> 1;
        const CUtensorMap* map = is_v ? &mapV : &mapK;
        const int col = (is_v ? p.v_col0 : p.k_col0) + h * kHd;
        uint8_t* dst = sKV + stage * kTileBytes;
        mbar_arrive_expect_tx(&kv_full[stage], kTileBytes);
        tma_load_3d(dst, map, &kv_full[stage], col, j * kTile, b);
        tma_load_3d(dst + kHalfBytes, map, &kv_full[stage], col + 64, j * kTile, b);
        ++issued;
      }
      mbar_wait(q_full, 0, p.err);
      for (int s = 0; s < kStages; ++s) {
        const int n_s = issued / kStages + (s < issued % kStages ? 1 : 0);
        if (n_s > 0) mbar_wait(&kv_full[s], static_cast<uint32_t>((n_s - 1) & 1), p.err);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_bf16_f32(kTile, kTile, 0, 0);
      const uint32_t idesc_pv = idesc_bf16_f32(kTile, kHd, 0, 1);
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t kv_addr = smem_u32(sKV);
      const uint32_t p_addr = smem_u32(sP);
      bool ok = mbar_wait(q_full, 0, p.err);
      auto issue_pv = [&](int i) -> bool {
        const int ld = 2 * i + 1;
        const int stage = ld % kStages;
        if (!mbar_wait(&p_full[i & 1], static_cast<uint32_t>((i >> 1) & 1), p.err)) return false;
        if (!mbar_wait(&kv_full[stage], static_cast<uint32_t>((ld / kStages) & 1), p.err)) return false;
        tc_fence_after();
        const uint32_t pa = p_addr + (i & 1) * kTileBytes;
        const uint32_t va = kv_addr + stage * kTileBytes;
#pragma unroll
        for (int k = 0; k < kTile / 16; ++k) {
          const uint64_t ad = sdesc_sw128(pa + (k >> 2) * kHalfBytes + (k & 3) * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(va + k * 16 * 128, kHalfBytes, 1024);
          tc_mma_bf16(tmem_o, ad, bd, idesc_pv, (i > 0 || k > 0) ? 1u : 0u);
        }
        tc_commit(&kv_empty[stage]);
        tc_commit(&o_done[i & 1]);
        return true;
      };
      for (int j = 0; ok && j < nkv; ++j) {
        const int ld = 2 * j;
        const int stage = ld % kStages;
        if (!mbar_wait(&kv_full[stage], static_cast<uint32_t>((ld / kStages) & 1), p.err)) break;
        if (!mbar_wait(&s_free[j & 1], static_cast<uint32_t>(((j >> 1) & 1) ^ 1), p.err)) break;
        tc_fence_after();
        const uint32_t s_tmem = tmem_base + (j & 1) * kTile;
        const uint32_t ka = kv_addr + stage * kTileBytes;
#pragma unroll
        for (int k = 0; k < kHd / 16; ++k) {
          const uint32_t off = (k >> 2) * kHalfBytes + (k & 3) * 32;
          tc_mma_bf16(s_tmem, sdesc_sw128(q_addr + off, 16, 1024), sdesc_sw128(ka + off, 16, 1024), idesc_qk,
                      k > 0 ? 1u : 0u);
        }
        tc_commit(&kv_empty[stage]);
        tc_commit(&s_full[j & 1]);
        if (j > 0) ok = issue_pv(j - 1);
      }
      if (ok && nkv > 0) issue_pv(nkv - 1);
      tc_commit(drain);
      mbar_wait(drain, 0, p.err);
    }
  } else {
    // Softmax warps: TMEM lane quarter (warp % 4) holds query rows 32*quarter + lane.
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY;
    float l_run = 0.f;
    bool ok = true;
    for (int j = 0; ok && j < nkv; ++j) {
      if (!mbar_wait(&s_full[j & 1], static_cast<uint32_t>((j >> 1) & 1), p.err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[kTile];
      {
        const uint32_t sa = tmem_base + lane_off + (j & 1) * kTile;
#pragma unroll
        for (int c = 0; c < kTile / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(sa + c * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(r[i]);
        }
      }
      tc_fence_before();
      mbar_arrive(&s_free[j & 1]);
      const int valid = p.Lk - j * kTile;
      if (valid < kTile) {
#pragma unroll
        for (int i = 0; i < kTile; ++i)
          if (i >= valid) s[i] = -INFINITY;
      }
      float mx = s[0];
#pragma unroll
      for (int i = 1; i < kTile; ++i) mx = fmaxf(mx, s[i]);
      if (j == 0) {
        m_run = mx;
      } else if ((mx - m_run) * sl2 > kRescaleLog2) {
        // O must hold P_{j-1} V_{j-1} before it is rescaled.
        if (!mbar_wait(&o_done[(j - 1) & 1], static_cast<uint32_t>(((j - 1) >> 1) & 1), p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float alpha = ex2_approx((m_run - mx) * sl2);
#pragma unroll
        for (int c = 0; c < kHd / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tmem_o + lane_off + c * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tmem_st32(tmem_o + lane_off + c * 32, r);
        }
        tmem_st_wait();
        l_run *= alpha;
        m_run = mx;
      }
      const float nb = -m_run * sl2;
      float rs = 0.f;
#pragma unroll
      for (int i = 0; i < kTile; ++i) {
        s[i] = ex2_approx(fmaf(s[i], sl2, nb));
        rs += s[i];
      }
      l_run += rs;
      // The P buffer of this parity was last read by PV_{j-2}.
      if (j >= 2 && !mbar_wait(&o_done[j & 1], static_cast<uint32_t>(((j - 2) >> 1) & 1), p.err)) {
        ok = false;
        break;
      }
      uint8_t* prow = sP + (j & 1) * kTileBytes + row * 128;
#pragma unroll
      for (int c16 = 0; c16 < kTile / 8; ++c16) {
        const int half = c16 >> 3, ch = c16 & 7;
        uint4 u;
        u.x = pack_bf16x2(s[c16 * 8 + 0], s[c16 * 8 + 1]);
        u.y = pack_bf16x2(s[c16 * 8 + 2], s[c16 * 8 + 3]);
        u.z = pack_bf16x2(s[c16 * 8 + 4], s[c16 * 8 + 5]);
        u.w = pack_bf16x2(s[c16 * 8 + 6], s[c16 * 8 + 7]);
        *reinterpret_cast<uint4*>(prow + half * kHalfBytes + ((ch ^ (row & 7)) << 4)) = u;
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[j & 1]);
    }
    if (ok && nkv > 0) {
      const int last = nkv - 1;
      if (mbar_wait(&o_done[last & 1], static_cast<uint32_t>((last >> 1) & 1), p.err)) {
        tc_fence_after();
        const float inv = 1.0f / l_run;
        const int grow = q0 + row;
        __nv_bfloat16* orow = p.o + static_cast<int64_t>(b) * p.o_batch_stride +
                              static_cast<int64_t>(grow) * p.o_row_stride + p.o_col0 + h * kHd;
#pragma unroll
        for (int c = 0; c < kHd / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tmem_o + lane_off + c * 32, r);
          tmem_ld_wait();
          if (grow < p.Lq) {
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              uint4 u;
              u.x = pack_bf16x2(__uint_as_float(r[g * 8 + 0]) * inv, __uint_as_float(r[g * 8 + 1]) * inv);
              u.y = pack_bf16x2(__uint_as_float(r[g * 8 + 2]) * inv, __uint_as_float(r[g * 8 + 3]) * inv);
              u.z = pack_bf16x2(__uint_as_float(r[g * 8 + 4]) * inv, __uint_as_float(r[g * 8 + 5]) * inv);
              u.w = pack_bf16x2(__uint_as_float(r[g * 8 + 6]) * inv, __uint_as_float(r[g * 8 + 7]) * inv);
              reinterpret_cast<uint4*>(orow + c * 32)[g] = u;
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

bool make_operand_map(CUtensorMap* map, const AttnOperand& op, int B, int L) {
  const uint64_t dims[3] = {static_cast<uint64_t>(op.row_stride), static_cast<uint64_t>(L),
                            static_cast<uint64_t>(B)};
  const uint64_t strides[2] = {static_cast<uint64_t>(op.row_stride) * 2,
                               static_cast<uint64_t>(op.row_stride) * 2 * static_cast<uint64_t>(L)};
  const uint32_t box[3] = {64, kTile, 1};
  return make_tmap_bf16(map, op.ptr, 3, dims, strides, box);
}

}  // namespace

int launch_attn_tc(AttnOperand q, AttnOperand k, AttnOperand v, void* o, int64_t o_row_stride, int o_col0, int B,
                   int H, int Lq, int Lk, cudaStream_t s) {
  if (B == 0 || Lq == 0) return WAN_OK;
  if (Lk <= 0) return WAN_ERR_SHAPE;
  if (q.row_stride % 8 || k.row_stride % 8 || v.row_stride % 8 || o_row_stride % 8) return WAN_ERR_ALIGN;
  if (q.col0 % 8 || k.col0 % 8 || v.col0 % 8 || o_col0 % 8) return WAN_ERR_ALIGN;
  CUtensorMap mq, mk, mv;
  if (!make_operand_map(&mq, q, B, Lq) || !make_operand_map(&mk, k, B, Lk) || !make_operand_map(&mv, v, B, Lk))
    return WAN_ERR_CUDA;
  AttnParams p;
  p.Lq = Lq;
  p.Lk = Lk;
  p.H = H;
  p.q_col0 = q.col0;
  p.k_col0 = k.col0;
  p.v_col0 = v.col0;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(kHd)));
  p.o = static_cast<__nv_bfloat16*>(o);
  p.o_row_stride = o_row_stride;
  p.o_batch_stride = o_row_stride * Lq;
  p.o_col0 = o_col0;
  p.err = device_error_flag();
  static std::once_flag once[64];
  int dev = 0;
  cudaGetDevice(&dev);
  std::call_once(once[dev & 63], [] {
    cudaFuncSetAttribute(attn_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(kAttnSmem));
  });
  dim3 grid((Lq + kTile - 1) / kTile, H, B);
  trace_launch_begin(WAN_KIND_ATTN, s, 4.0 * B * H * static_cast<double>(Lq) * Lk * kHd);
  attn_fwd_tc_kernel<<<grid, kAttnThreads, kAttnSmem, s>>>(mq, mk, mv, p);
  int st = check_launch();
  trace_launch_end(WAN_KIND_ATTN, s);
  return st;
}

}  // namespace wan
