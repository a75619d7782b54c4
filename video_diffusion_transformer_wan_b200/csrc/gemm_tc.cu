// Kernel (c): persistent bf16 GEMM on the sm_100a tensor cores (tcgen05), computing
// out = epilogue(A W^T + bias) for the DiT's Linear layers: the fused QKV projection,
// the attention output projections with the gated residual, the FFN (GELU-tanh into
// the hidden, gated residual out of it), the patchify projection (fp32 store) and the
// head (scatter straight into the unpatchified latent).
//
// Tile 128 x BN x 64. One CTA per SM loops over output tiles:
//   warp 0  : TMA producer, a ring of kStages (A, W) stages with 128-byte swizzle;
//   warp 1  : one elected thread issues tcgen05.mma (M=128, N=BN, K=16) into a TMEM
//             accumulator; two accumulators alternate so the epilogue of one tile
//             overlaps the main loop of the next;
//   warps 2-9: epilogue; warp w reads TMEM lanes 32*(w%4).. (rows of the tile) and one
//             half of the tile's columns with tcgen05.ld, applies bias / activation /
//             scale and writes global memory. The gated fp32 residual and the fp32
//             store (their own instantiation) go through a 32x32 shared-memory block
//             per warp so that the read-modify-write of x, or the store, moves whole
//             128-byte row segments; with the thread-per-row layout of the TMEM load
//             it took 32 half-used sectors per instruction, the epilogue of the D x D
//             projections did not hide under their short main loop, and the patchify
//             projection (K = 64, nearly all epilogue) stored at a quarter of the HBM
//             bandwidth.
//
// Tile order: the row blocks are cut into groups of group_m; within a group the row
// block varies fastest, so the 148 tiles in flight share a slab of at most
// group_m row blocks of A (sized to stay in L2) and a few column blocks of W, and each
// operand comes from DRAM about once per group instead of once per wave.
#include <cuda_bf16.h>

#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace wan {
namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kEpiWarps = 8;
constexpr int kGemmThreads = 64 + 32 * kEpiWarps;
#ifndef WAN_GEMM_SLAB_MB
#define WAN_GEMM_SLAB_MB 32  // bytes of A (MiB) one tile group keeps resident in L2
#endif

template <int BN, bool kRes = false>
struct GemmCfg {
  static constexpr int kStages = BN == 256 ? 4 : (BN == 128 ? 6 : 8);
  static constexpr int kABytes = kBM * 128;  // 128-byte rows: 64 bf16 or 128 E4M3 elements
  static constexpr int kBBytes = BN * 128;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTmemCols = 2 * BN;
  // gated-residual instantiation: a 32x32 fp32 staging block per epilogue warp
  static constexpr size_t kEpiStageBytes = kRes ? static_cast<size_t>(kEpiWarps) * 32 * 32 * 4 : 0;
  static constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(kStages) * kStageBytes + 256 + kEpiStageBytes;
};

struct GemmParams {
  int M, N, K;
  int k_blocks;
  int wk_period_blocks;  // > 0: W column block = k block mod this
  int m_blocks, n_blocks;
  int group_m;           // row blocks per tile group
  int bk;                // elements of K per stage (64 bf16, 128 E4M3)
  const float* a_scale;  // E4M3: per-row scale of A (acc * a_scale[m] * w_scale[0]), else NULL
  const float* w_scale;
  const __nv_bfloat16* bias;
  void* out;
  GemmEpi epi;
  int* err;
};

__device__ __forceinline__ float gelu_tanh_f(float v) {
  const float u = 0.7978845608028654f * (v + 0.044715f * v * v * v);
  return 0.5f * v * (1.0f + tanh_approx(u));
}

// Output tile -> (row block, column block), row block fastest within a group.
__device__ __forceinline__ void tile_coords(const GemmParams& p, int tile, int& mb, int& nb) {
  const int per_group = p.group_m * p.n_blocks;
  const int g = tile / per_group;
  const int r = tile - g * per_group;
  const int m_first = g * p.group_m;
  const int gm = min(p.group_m, p.m_blocks - m_first);
  mb = m_first + r % gm;
  nb = r / gm;
}

// Apply the epilogue to 32 consecutive accumulator columns [n0, n0+32) of one row.
__device__ __forceinline__ void epilogue_chunk(const GemmParams& p, int row, int n0, const uint32_t (&r)[32]) {
  if (row >= p.M || n0 >= p.N) return;
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
  if (p.a_scale) {
    const float sc = __ldg(p.a_scale + row) * __ldg(p.w_scale);
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] *= sc;
  }
  const bool full = n0 + 32 <= p.N;
  if (p.bias) {
    if (full) {
      const uint4* bp = reinterpret_cast<const uint4*>(p.bias + n0);
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        uint4 u = __ldg(bp + g);
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float2 f = __bfloat1622float2(h[j]);
          v[g * 8 + 2 * j] += f.x;
          v[g * 8 + 2 * j + 1] += f.y;
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (n0 + i < p.N) v[i] += __bfloat162float(p.bias[n0 + i]);
    }
  }
  const int kind = p.epi.kind;
  if (kind == WAN_EPI_STORE || kind == WAN_EPI_GELU || kind == kEpiSeqScatter) {
    if (kind == WAN_EPI_GELU) {
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = gelu_tanh_f(v[i]);
    }
    __nv_bfloat16* o;
    if (kind == kEpiSeqScatter) {
      // The 32 columns lie inside one head, hence inside one destination rank's slab.
      const int b = row / p.epi.sp_rows_local, i = row - b * p.epi.sp_rows_local;
      const int part = n0 / p.epi.sp_part_cols, c = n0 - part * p.epi.sp_part_cols;
      const int s = c / p.epi.sp_rank_cols;
      const int64_t drow = static_cast<int64_t>(b) * p.epi.sp_rows_total + p.epi.sp_row_off + i;
      o = static_cast<__nv_bfloat16*>(p.epi.sp_dst[s]) + drow * p.epi.ldo + part * p.epi.sp_rank_cols +
          (c - s * p.epi.sp_rank_cols);
    } else {
      o = static_cast<__nv_bfloat16*>(p.out) + static_cast<int64_t>(row) * p.epi.ldo + n0;
    }
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      if (n0 + g * 8 < p.N) {
        uint4 u;
        u.x = pack_bf16x2(v[g * 8 + 0], v[g * 8 + 1]);
        u.y = pack_bf16x2(v[g * 8 + 2], v[g * 8 + 3]);
        u.z = pack_bf16x2(v[g * 8 + 4], v[g * 8 + 5]);
        u.w = pack_bf16x2(v[g * 8 + 6], v[g * 8 + 7]);
        reinterpret_cast<uint4*>(o)[g] = u;
      }
    }
  } else if (kind == WAN_EPI_F32) {
    float* o = static_cast<float*>(p.out) + static_cast<int64_t>(row) * p.epi.ldo + n0;
#pragma unroll
    for (int g = 0; g < 8; ++g)
      if (n0 + g * 4 < p.N)
        reinterpret_cast<float4*>(o)[g] = make_float4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
  } else if (kind == kEpiHeadScatter) {  // n = c*4 + ph*2 + pw, row = b*L + (f*Hh + i)*Wh + j
    const int L = p.epi.rows_per_batch;
    const int b = row / L, l = row % L;
    const int Hh = p.epi.sc_H / 2, Wh = p.epi.sc_W / 2;
    const int f = l / (Hh * Wh), ii = (l / Wh) % Hh, jj = l % Wh;
    float* o = static_cast<float*>(p.out);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int n = n0 + i;
      if (n < p.N) {
        const int c = n >> 2, ph = (n >> 1) & 1, pw = n & 1;
        const int64_t idx = ((static_cast<int64_t>(b) * p.epi.sc_C + c) * p.epi.sc_F + f) * p.epi.sc_H * p.epi.sc_W +
                            static_cast<int64_t>(2 * ii + ph) * p.epi.sc_W + (2 * jj + pw);
        o[idx] = v[i];
      }
    }
  }
}

// bf16 store (plain or GELU) of one 32x32 block through shared memory: thread = row
// applies scale, bias and GELU to its 32 columns, packs them to bf16 and stages the
// 64-byte row (16-byte units XOR-swizzled by row); the warp then reads it back eight
// rows per instruction (4 threads x 16 bytes per row), so each global store moves
// whole 64-byte row segments instead of one 16-byte piece of 32 rows.
__device__ __forceinline__ void store_staged_bf16(const GemmParams& p, uint32_t* stg, int r0, int n0, int lane,
                                                  const uint32_t (&r)[32]) {
  const int row = r0 + lane;
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
  if (p.a_scale) {
    const float sc = row < p.M ? __ldg(p.a_scale + row) * __ldg(p.w_scale) : 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] *= sc;
  }
  if (p.bias) {
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      if (n0 + g * 8 < p.N) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(p.bias + n0) + g);
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = __bfloat1622float2(h[j]);
          v[g * 8 + 2 * j] += f.x;
          v[g * 8 + 2 * j + 1] += f.y;
        }
      }
    }
  }
  if (p.epi.kind == WAN_EPI_GELU) {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = gelu_tanh_f(v[i]);
  }
  const int swz = (lane >> 1) & 3;
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    uint4 u;
    u.x = pack_bf16x2(v[g * 8 + 0], v[g * 8 + 1]);
    u.y = pack_bf16x2(v[g * 8 + 2], v[g * 8 + 3]);
    u.z = pack_bf16x2(v[g * 8 + 4], v[g * 8 + 5]);
    u.w = pack_bf16x2(v[g * 8 + 6], v[g * 8 + 7]);
    reinterpret_cast<uint4*>(stg + lane * 16)[g ^ swz] = u;
  }
  __syncwarp();
  const int q = lane & 3;
  const int gcol = n0 + q * 8;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int rr = i * 8 + (lane >> 2);
    const int grow = r0 + rr;
    const uint4 u = reinterpret_cast<const uint4*>(stg + rr * 16)[q ^ ((rr >> 1) & 3)];
    if (grow < p.M && gcol < p.N)
      *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + static_cast<int64_t>(grow) * p.epi.ldo + gcol) = u;
  }
  __syncwarp();
}

// Gated residual (and plain fp32 store) epilogue through shared memory: for each
// 32-column chunk the warp reads its 32 rows from TMEM (thread = row), scales and adds
// the bias, stages the 32x32 block (16-byte units XOR-swizzled by row), then reads it
// back four rows per instruction (8 threads x 16 bytes per row) so that every fp32
// read-modify-write of x (or store of the fp32 output) moves whole 128-byte row
// segments.
__device__ __forceinline__ void residual_staged(const GemmParams& p, float* stg, uint32_t t_row, int r0, int n0,
                                                int lane, int chunks) {
  const int row = r0 + lane;
  const float sc = p.a_scale ? (row < p.M ? __ldg(p.a_scale + row) : 0.f) * __ldg(p.w_scale) : 1.0f;
  const int sub = lane >> 3, cq = lane & 7;
  const bool residual = p.epi.kind == WAN_EPI_RESIDUAL;
#pragma unroll 1
  for (int c = 0; c < chunks; ++c) {
    const int col0 = n0 + c * 32;
    uint32_t r[32];
    tmem_ld32(t_row + c * 32, r);
    tmem_ld_wait();
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float4 v = make_float4(__uint_as_float(r[4 * k]) * sc, __uint_as_float(r[4 * k + 1]) * sc,
                             __uint_as_float(r[4 * k + 2]) * sc, __uint_as_float(r[4 * k + 3]) * sc);
      if (p.bias && col0 + 4 * k < p.N) {
        const uint2 u = __ldg(reinterpret_cast<const uint2*>(p.bias + col0 + 4 * k));
        const float2 b01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
        const float2 b23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
        v.x += b01.x; v.y += b01.y; v.z += b23.x; v.w += b23.y;
      }
      reinterpret_cast<float4*>(stg + lane * 32)[k ^ (lane & 7)] = v;
    }
    __syncwarp();
    const int gcol = col0 + cq * 4;
    if (!residual) {  // fp32 store
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int rr = i * 4 + sub;
        const int grow = r0 + rr;
        if (grow < p.M && gcol < p.N)
          *reinterpret_cast<float4*>(static_cast<float*>(p.out) + static_cast<int64_t>(grow) * p.epi.ldo + gcol) =
              reinterpret_cast<const float4*>(stg + rr * 32)[cq ^ (rr & 7)];
      }
      __syncwarp();
      continue;
    }
    float4 gb = make_float4(0.f, 0.f, 0.f, 0.f);
    if (p.epi.gate_bias && gcol < p.N) gb = __ldg(reinterpret_cast<const float4*>(p.epi.gate_bias + gcol));
    float4 x[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int grow = r0 + i * 4 + sub;
      if (grow < p.M && gcol < p.N)
        x[i] = *reinterpret_cast<const float4*>(static_cast<const float*>(p.out) + static_cast<int64_t>(grow) * p.epi.ldo +
                                                gcol);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int rr = i * 4 + sub;
      const int grow = r0 + rr;
      if (grow < p.M && gcol < p.N) {
        const float4 v = reinterpret_cast<const float4*>(stg + rr * 32)[cq ^ (rr & 7)];
        float4 g = make_float4(1.f, 1.f, 1.f, 1.f);
        if (p.epi.gate) {
          g = __ldg(reinterpret_cast<const float4*>(
              p.epi.gate + static_cast<int64_t>(grow / p.epi.rows_per_batch) * p.epi.gate_bstride + gcol));
          if (p.epi.gate_bias) {
            g.x += gb.x; g.y += gb.y; g.z += gb.z; g.w += gb.w;
          }
        }
        float4 o = x[i];
        o.x += g.x * v.x; o.y += g.y * v.y; o.z += g.z * v.z; o.w += g.w * v.w;
        *reinterpret_cast<float4*>(static_cast<float*>(p.out) + static_cast<int64_t>(grow) * p.epi.ldo + gcol) = o;
      }
    }
    __syncwarp();
  }
}

// Gated residual (or fp32 store) by bulk tensor operations: for each 32-column chunk the
// warp reads its 32 rows from TMEM (thread = row), forms g * (acc * scale + bias) (or
// acc * scale + bias for the store), stages the 32 x 32 fp32 block in the 128-byte
// swizzled layout of the x tensor map, and one lane issues a bulk reduce-add of the
// block into x (x += block, element-wise in L2) or a bulk store. x is never read into
// the SM. Each x element is updated by exactly one tile, so the result does not depend
// on timing. The block is rewritten only after the previous bulk operation read it.
__device__ __forceinline__ void residual_tma(const GemmParams& p, const CUtensorMap* map_x, float* stg,
                                             uint32_t t_row, int r0, int n0, int lane, int chunks) {
  const int row = r0 + lane;
  const float sc = p.a_scale ? (row < p.M ? __ldg(p.a_scale + row) : 0.f) * __ldg(p.w_scale) : 1.0f;
  const bool residual = p.epi.kind == WAN_EPI_RESIDUAL;
  const float* gate_row = residual && p.epi.gate
                              ? p.epi.gate + static_cast<int64_t>(min(row, p.M - 1) / p.epi.rows_per_batch) *
                                                 p.epi.gate_bstride
                              : nullptr;
#pragma unroll 1
  for (int c = 0; c < chunks; ++c) {
    const int col0 = n0 + c * 32;
    uint32_t r[32];
    tmem_ld32(t_row + c * 32, r);
    if (lane == 0) bulk_wait_read_all();
    tmem_ld_wait();
    __syncwarp();
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int col = col0 + 4 * k;
      float4 v = make_float4(__uint_as_float(r[4 * k]) * sc, __uint_as_float(r[4 * k + 1]) * sc,
                             __uint_as_float(r[4 * k + 2]) * sc, __uint_as_float(r[4 * k + 3]) * sc);
      if (col < p.N) {
        if (p.bias) {
          const uint2 u = __ldg(reinterpret_cast<const uint2*>(p.bias + col));
          const float2 b01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
          const float2 b23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
          v.x += b01.x; v.y += b01.y; v.z += b23.x; v.w += b23.y;
        }
        if (gate_row) {
          float4 g = __ldg(reinterpret_cast<const float4*>(gate_row + col));
          if (p.epi.gate_bias) {
            const float4 gb = __ldg(reinterpret_cast<const float4*>(p.epi.gate_bias + col));
            g.x += gb.x; g.y += gb.y; g.z += gb.z; g.w += gb.w;
          }
          v.x *= g.x; v.y *= g.y; v.z *= g.z; v.w *= g.w;
        }
      }
      reinterpret_cast<float4*>(stg + lane * 32)[k ^ (lane & 7)] = v;
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0 && r0 < p.M && col0 < p.N) {  // the tensor map clips the block at M and N
      if (residual)
        tma_reduce_add_2d(map_x, stg, col0, r0);
      else
        tma_store_2d(map_x, stg, col0, r0);
      bulk_commit_group();
    }
  }
}

template <int BN, bool kF8, bool kRes>
__device__ __forceinline__ void gemm_body(const CUtensorMap& mapA, const CUtensorMap& mapB, const GemmParams& p) {
  using C = GemmCfg<BN, kRes>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::kStages * C::kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + C::kStages * C::kBBytes);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  float* epi_stage = reinterpret_cast<float*>(sB + C::kStages * C::kBBytes + 256);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 32 * kEpiWarps);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mapA);
    tma_prefetch_desc(&mapB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int num_tiles = p.m_blocks * p.n_blocks;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int64_t issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        int mb, nb;
        tile_coords(p, tile, mb, nb);
        const int m0 = mb * kBM;
        const int n0 = nb * BN;
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, p.err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], C::kStageBytes);
          const int kbw = p.wk_period_blocks > 0 ? kb % p.wk_period_blocks : kb;
          tma_load_2d(sA + stage * C::kABytes, &mapA, &full[stage], kb * p.bk, m0);
          tma_load_2d(sB + stage * C::kBBytes, &mapB, &full[stage], kbw * p.bk, n0);
          ++issued;
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Drain: every issued tile load has landed before the CTA exits.
      for (int s = 0; s < C::kStages; ++s) {
        const int64_t n_s = issued / C::kStages + (s < issued % C::kStages ? 1 : 0);
        if (n_s > 0) mbar_wait(&full[s], static_cast<uint32_t>((n_s - 1) & 1), p.err);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = kF8 ? idesc_e4m3_f32(kBM, BN) : idesc_bf16_f32(kBM, BN, 0, 0);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int it = 0;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x, ++it) {
        const int acc = it & 1;
        if (!mbar_wait(&tempty[acc], ((it >> 1) & 1) ^ 1u, p.err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait(&full[stage], phase, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * C::kABytes);
          const uint32_t b_addr = smem_u32(sB + stage * C::kBBytes);
#pragma unroll
          for (int k = 0; k < 4; ++k) {  // 32 bytes of K per MMA: 16 bf16 or 32 E4M3
            const uint64_t ad = sdesc_sw128(a_addr + k * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(b_addr + k * 32, 16, 1024);
            if (kF8)
              tc_mma_e4m3(d_tmem, ad, bd, idesc, (kb | k) != 0 ? 1u : 0u);
            else
              tc_mma_bf16(d_tmem, ad, bd, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          tc_commit(&empty[stage]);
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) tc_commit(&tfull[acc]);
      }
      // Drain: all issued MMAs complete before TMEM is released.
      tc_commit(drain);
      mbar_wait(drain, 0, p.err);
    }
  } else {
    const int quarter = warp & 3;           // TMEM lanes 32*quarter .. (rows of the tile)
    const int colhalf = (warp - 2) >> 2;    // which half of the tile's columns
    constexpr int kMine = BN / 64;          // 32-column chunks per warp
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int acc = it & 1;
      if (!mbar_wait_warp(&tfull[acc], (it >> 1) & 1, p.err)) break;
      tc_fence_after();
      int mb, nb;
      tile_coords(p, tile, mb, nb);
      const int m0 = mb * kBM;
      const int n0 = nb * BN + colhalf * (BN / 2);
      const int row = m0 + quarter * 32 + lane;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                             static_cast<uint32_t>(acc * BN + colhalf * (BN / 2));
      if constexpr (kRes) {
        residual_staged(p, epi_stage + (warp - 2) * 1024, t_row, m0 + quarter * 32, n0, lane, kMine);
      } else {
#pragma unroll 1
        for (int c = 0; c < kMine; c += 2) {
          uint32_t r0[32], r1[32];
          tmem_ld32(t_row + c * 32, r0);
          if (c + 1 < kMine) tmem_ld32(t_row + (c + 1) * 32, r1);
          tmem_ld_wait();
          epilogue_chunk(p, row, n0 + c * 32, r0);
          if (c + 1 < kMine) epilogue_chunk(p, row, n0 + (c + 1) * 32, r1);
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

template <int BN, bool kRes>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_bf16_tc_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                        const GemmParams p) {
  gemm_body<BN, false, kRes>(mapA, mapB, p);
}

template <int BN, bool kRes>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_e4m3_tc_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                        const GemmParams p) {
  gemm_body<BN, true, kRes>(mapA, mapB, p);
}

// ---------------------------------------------------------------- CTA-pair GEMM
// bf16 GEMMs with N >= 256 on CTA pairs: a pair owns a 256 x 256 output tile; CTA r of
// the pair loads rows [128 r, 128 r + 128) of the tile's A and of its W block (W rows =
// output columns) into the same shared-memory offsets, and the even CTA's MMA thread
// issues tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16), which reads both CTAs'
// halves and leaves each CTA's 128 accumulator rows (all 256 columns) in its own TMEM.
// Per SM and k-block of 64 this moves 32 KB into shared memory instead of 48 KB (the
// 128 x 256 one-SM tile loads all of its 256 W rows), for the same FLOPs.
// Barriers: each CTA's TMA loads complete on the even CTA's full[stage] (only the even
// CTA's producer arms it, with both CTAs' bytes); the MMA commits release empty[stage]
// and signal tfull[acc] in both CTAs; both CTAs' epilogue warps release tempty[acc] on
// the even CTA. Barriers are initialised, and TMEM allocated, in both CTAs before a
// cluster barrier; a second one precedes deallocation.
// Epilogue: the gated residual and the fp32 store stage fp32 blocks and hand them to
// bulk tensor operations (residual_tma: a reduce-add into x, or a store), so x is never
// read into the SM; the bf16 store and GELU stage bf16 blocks (store_staged_bf16), so
// each store moves 64-byte row segments.
#ifndef WAN_PAIR_STAGES_PLAIN
#define WAN_PAIR_STAGES_PLAIN 6  // ring depth of the pair kernel without the gated residual
#endif
constexpr int kPairStageBytes = 2 * kBM * 128;  // A half + W half: 128 rows x 128 bytes each
template <bool kRes>
struct PairCfg {
  static constexpr int kStages = kRes ? 6 : WAN_PAIR_STAGES_PLAIN;
  // fp32 32x32 block per epilogue warp (gated residual), or a bf16 one (staged store)
  static constexpr size_t kEpiStageBytes = static_cast<size_t>(kEpiWarps) * 32 * 32 * (kRes ? 4 : 2);
  static constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(kStages) * kPairStageBytes + 256 + kEpiStageBytes;
};

template <bool kF8, bool kRes>
__device__ __forceinline__ void gemm_pair_body(const CUtensorMap& mapA, const CUtensorMap& mapB, const CUtensorMap& mapX,
                                               const GemmParams& p) {
  constexpr int kPairStages = PairCfg<kRes>::kStages;
  constexpr int kHalf = kBM * 128;  // bytes of one 128-row operand half per stage
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kPairStages * kHalf;
  // epilogue staging (1024-byte aligned, as the x tensor map's 128-byte swizzle needs),
  // then the barriers
  float* epi_stage = reinterpret_cast<float*>(sB + kPairStages * kHalf);
  uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(epi_stage) + PairCfg<kRes>::kEpiStageBytes);
  uint64_t* empty = full + kPairStages;
  uint64_t* tfull = empty + kPairStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  const int num_tiles = p.m_blocks * p.n_blocks;
  if (threadIdx.x == 0) {
    for (int st = 0; st < kPairStages; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * 32 * kEpiWarps);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mapA);
    tma_prefetch_desc(&mapB);
    if (kRes) tma_prefetch_desc(&mapX);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // The even CTA's barriers, as shared::cluster addresses.
  const uint32_t full0 = mapa_shared(smem_u32(full), 0);
  const uint32_t tempty0 = mapa_shared(smem_u32(tempty), 0);

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int64_t issued = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < num_tiles; tile += npairs) {
        int mb, nb;
        tile_coords(p, tile, mb, nb);
        const int m0 = mb * 2 * kBM + static_cast<int>(rank) * kBM;
        const int n0 = nb * 2 * kBM + static_cast<int>(rank) * kBM;
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, p.err)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * kPairStageBytes);
          const int kbw = p.wk_period_blocks > 0 ? kb % p.wk_period_blocks : kb;
          const uint32_t bar = full0 + static_cast<uint32_t>(stage) * 8u;
          tma_load_2d_pair(sA + stage * kHalf, &mapA, bar, kb * p.bk, m0);
          tma_load_2d_pair(sB + stage * kHalf, &mapB, bar, kbw * p.bk, n0);
          ++issued;
          if (++stage == kPairStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Drain: each slot's last load was consumed (the MMA's release reaches both CTAs),
      // so no copy into this CTA's shared memory is in flight at exit.
      for (int st = 0; st < kPairStages; ++st) {
        const int64_t n_s = issued / kPairStages + (st < issued % kPairStages ? 1 : 0);
        if (n_s > 0) mbar_wait(&empty[st], static_cast<uint32_t>((n_s - 1) & 1), p.err);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      const uint32_t idesc = kF8 ? idesc_e4m3_f32(2 * kBM, 2 * kBM) : idesc_bf16_f32(2 * kBM, 2 * kBM, 0, 0);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int it = 0;
      for (int tile = pair; ok && tile < num_tiles; tile += npairs, ++it) {
        const int acc = it & 1;
        if (!mbar_wait(&tempty[acc], ((it >> 1) & 1) ^ 1u, p.err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * 256);
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait(&full[stage], phase, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * kHalf);
          const uint32_t b_addr = smem_u32(sB + stage * kHalf);
#pragma unroll
          for (int k = 0; k < 4; ++k) {  // 32 bytes of K per MMA: 16 bf16 or 32 E4M3
            const uint64_t ad = sdesc_sw128(a_addr + k * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(b_addr + k * 32, 16, 1024);
            if constexpr (kF8)
              tc_mma_e4m3_pair(d_tmem, ad, bd, idesc, (kb | k) != 0 ? 1u : 0u);
            else
              tc_mma_bf16_pair(d_tmem, ad, bd, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          tc_commit_pair(&empty[stage], 0x3);
          if (++stage == kPairStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) tc_commit_pair(&tfull[acc], 0x3);
      }
      tc_commit_pair(drain, 0x1);
      mbar_wait(drain, 0, p.err);
    }
  } else {
    const int quarter = warp & 3;           // TMEM lanes 32*quarter .. (rows of this CTA's half)
    const int colhalf = (warp - 2) >> 2;    // which 128 of the tile's 256 columns
    constexpr int kMine = 4;                // 32-column chunks per warp
    int it = 0;
    for (int tile = pair; tile < num_tiles; tile += npairs, ++it) {
      const int acc = it & 1;
      if (!mbar_wait_warp(&tfull[acc], (it >> 1) & 1, p.err)) break;
      tc_fence_after();
      int mb, nb;
      tile_coords(p, tile, mb, nb);
      const int m0 = mb * 2 * kBM + static_cast<int>(rank) * kBM;
      const int n0 = nb * 2 * kBM + colhalf * kBM;
      const int row = m0 + quarter * 32 + lane;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                             static_cast<uint32_t>(acc * 256 + colhalf * kBM);
      if constexpr (kRes) {
        residual_tma(p, &mapX, epi_stage + (warp - 2) * 1024, t_row, m0 + quarter * 32, n0, lane, kMine);
      } else if (p.epi.kind == WAN_EPI_STORE || p.epi.kind == WAN_EPI_GELU) {
        uint32_t* stg = reinterpret_cast<uint32_t*>(epi_stage) + (warp - 2) * 512;
#pragma unroll 1
        for (int c = 0; c < kMine; c += 2) {
          uint32_t r0[32], r1[32];
          tmem_ld32(t_row + c * 32, r0);
          tmem_ld32(t_row + (c + 1) * 32, r1);
          tmem_ld_wait();
          store_staged_bf16(p, stg, m0 + quarter * 32, n0 + c * 32, lane, r0);
          store_staged_bf16(p, stg, m0 + quarter * 32, n0 + (c + 1) * 32, lane, r1);
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < kMine; c += 2) {
          uint32_t r0[32], r1[32];
          tmem_ld32(t_row + c * 32, r0);
          tmem_ld32(t_row + (c + 1) * 32, r1);
          tmem_ld_wait();
          epilogue_chunk(p, row, n0 + c * 32, r0);
          epilogue_chunk(p, row, n0 + (c + 1) * 32, r1);
        }
      }
      tc_fence_before();
      mbar_arrive_cluster(tempty0 + static_cast<uint32_t>(acc) * 8u);
    }
  }
  // The epilogue's bulk operations have completed before the CTA can exit.
  if (kRes && warp >= 2 && lane == 0) bulk_wait_all();
  // Both CTAs are done with TMEM (and no remote arrival is pending) before it is freed.
  __syncwarp();
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

template <bool kRes>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    gemm_bf16_pair_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                          const __grid_constant__ CUtensorMap mapX, const GemmParams p) {
  gemm_pair_body<false, kRes>(mapA, mapB, mapX, p);
}

template <bool kRes>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    gemm_e4m3_pair_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                          const __grid_constant__ CUtensorMap mapX, const GemmParams p) {
  gemm_pair_body<true, kRes>(mapA, mapB, mapX, p);
}

// Launch one instantiation (the shared-memory opt-in is set once per device for each).
template <int BN, bool kF8, bool kRes>
int launch_inst(const CUtensorMap& mapA, const CUtensorMap& mapB, const GemmParams& p, int grid, cudaStream_t s) {
  using C = GemmCfg<BN, kRes>;
  auto kern = kF8 ? gemm_e4m3_tc_kernel<BN, kRes> : gemm_bf16_tc_kernel<BN, kRes>;
  static std::once_flag once[64];
  int dev = 0;
  cudaGetDevice(&dev);
  std::call_once(once[dev & 63],
                 [kern] { cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(C::kSmemBytes)); });
  kern<<<grid, kGemmThreads, C::kSmemBytes, s>>>(mapA, mapB, p);
  return check_launch();
}

int sm_count() {
  static int counts[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 148;
  if (counts[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    counts[dev] = n > 0 ? n : 148;
  }
  return counts[dev];
}

#ifndef WAN_GEMM_PAIR
#define WAN_GEMM_PAIR 1  // bf16 GEMMs with N >= 256, K >= 256, M >= 1024 on CTA pairs
#endif

// N >= 256: the CTA-pair kernels (256 x 256 tiles), bf16 or E4M3 operands.
template <bool kF8>
int launch_pair(const void* A, int64_t lda, const void* W, const void* bias, void* out, int M, int N, int K,
                int w_k_period, const GemmEpi& epi, cudaStream_t s, const float* a_scale = nullptr,
                const float* w_scale = nullptr) {
  constexpr int bk = kF8 ? 128 : 64;  // elements per 128-byte row
  constexpr int es = kF8 ? 1 : 2;
  CUtensorMap mapA, mapB;
  const uint64_t dimsA[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(M)};
  const uint64_t strA[1] = {static_cast<uint64_t>(lda) * es};
  const uint32_t box[2] = {static_cast<uint32_t>(bk), static_cast<uint32_t>(kBM)};
  const int kw = w_k_period > 0 ? w_k_period : K;
  const uint64_t dimsB[2] = {static_cast<uint64_t>(kw), static_cast<uint64_t>(N)};
  const uint64_t strB[1] = {static_cast<uint64_t>(kw) * es};
  const bool maps_ok = kF8 ? make_tmap_u8(&mapA, A, 2, dimsA, strA, box) && make_tmap_u8(&mapB, W, 2, dimsB, strB, box)
                           : make_tmap_bf16(&mapA, A, 2, dimsA, strA, box) &&
                                 make_tmap_bf16(&mapB, W, 2, dimsB, strB, box);
  if (!maps_ok) return WAN_ERR_CUDA;
  GemmParams p;
  p.M = M;
  p.N = N;
  p.K = K;
  p.bk = bk;
  p.k_blocks = (K + bk - 1) / bk;
  p.wk_period_blocks = w_k_period > 0 ? w_k_period / bk : 0;
  p.m_blocks = (M + 2 * kBM - 1) / (2 * kBM);
  p.n_blocks = (N + 2 * kBM - 1) / (2 * kBM);
  {
    const int64_t slab_rows = (static_cast<int64_t>(WAN_GEMM_SLAB_MB) << 20) / (static_cast<int64_t>(K) * es * 2 * kBM);
    p.group_m = static_cast<int>(slab_rows < 1 ? 1 : (slab_rows > p.m_blocks ? p.m_blocks : slab_rows));
  }
  p.a_scale = a_scale;
  p.w_scale = w_scale;
  p.bias = static_cast<const __nv_bfloat16*>(bias);
  p.out = out;
  p.epi = epi;
  p.err = device_error_flag();
  const int tiles = p.m_blocks * p.n_blocks;
  const int pairs = sm_count() / 2;
  const int grid = 2 * (tiles < pairs ? tiles : pairs);
  const bool staged = epi.kind == WAN_EPI_RESIDUAL || epi.kind == WAN_EPI_F32;
  // x (fp32, [M, ldo]) for the bulk reduce-add / store of the staged epilogue: 32 x 32
  // boxes; every box starts at a column that is a multiple of 32 (128 bytes).
  CUtensorMap mapX = mapA;
  if (staged) {
    const uint64_t dimsX[2] = {static_cast<uint64_t>(N), static_cast<uint64_t>(M)};
    const uint64_t strX[1] = {static_cast<uint64_t>(epi.ldo) * 4};
    const uint32_t boxX[2] = {32, 32};
    if (!make_tmap_f32(&mapX, out, 2, dimsX, strX, boxX)) return WAN_ERR_CUDA;
  }
  auto kern = staged ? (kF8 ? gemm_e4m3_pair_kernel<true> : gemm_bf16_pair_kernel<true>)
                     : (kF8 ? gemm_e4m3_pair_kernel<false> : gemm_bf16_pair_kernel<false>);
  const size_t smem = staged ? PairCfg<true>::kSmemBytes : PairCfg<false>::kSmemBytes;
  static std::once_flag once[2][64];
  int dev = 0;
  cudaGetDevice(&dev);
  std::call_once(once[staged ? 1 : 0][dev & 63],
                 [kern, smem] { cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                     static_cast<int>(smem)); });
  kern<<<grid, kGemmThreads, smem, s>>>(mapA, mapB, mapX, p);
  return check_launch();
}

template <int BN, bool kF8>
int launch_bn(const void* A, int64_t lda, const void* W, const void* bias, void* out, int M, int N, int K,
              int w_k_period, const GemmEpi& epi, cudaStream_t s, const float* a_scale = nullptr,
              const float* w_scale = nullptr) {
  constexpr int bk = kF8 ? 128 : 64;  // elements per 128-byte row
  constexpr int es = kF8 ? 1 : 2;
  CUtensorMap mapA, mapB;
  const uint64_t dimsA[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(M)};
  const uint64_t strA[1] = {static_cast<uint64_t>(lda) * es};
  const uint32_t boxA[2] = {bk, kBM};
  const int kw = w_k_period > 0 ? w_k_period : K;
  const uint64_t dimsB[2] = {static_cast<uint64_t>(kw), static_cast<uint64_t>(N)};
  const uint64_t strB[1] = {static_cast<uint64_t>(kw) * es};
  const uint32_t boxB[2] = {bk, BN};
  const bool maps_ok = kF8 ? make_tmap_u8(&mapA, A, 2, dimsA, strA, boxA) && make_tmap_u8(&mapB, W, 2, dimsB, strB, boxB)
                           : make_tmap_bf16(&mapA, A, 2, dimsA, strA, boxA) &&
                                 make_tmap_bf16(&mapB, W, 2, dimsB, strB, boxB);
  if (!maps_ok) return WAN_ERR_CUDA;
  GemmParams p;
  p.M = M;
  p.N = N;
  p.K = K;
  p.bk = bk;
  p.k_blocks = (K + bk - 1) / bk;
  p.wk_period_blocks = w_k_period > 0 ? w_k_period / bk : 0;
  p.m_blocks = (M + kBM - 1) / kBM;
  p.n_blocks = (N + BN - 1) / BN;
  {
    const int64_t slab_rows = (static_cast<int64_t>(WAN_GEMM_SLAB_MB) << 20) / (static_cast<int64_t>(K) * es * kBM);
    p.group_m = static_cast<int>(slab_rows < 1 ? 1 : (slab_rows > p.m_blocks ? p.m_blocks : slab_rows));
  }
  p.a_scale = a_scale;
  p.w_scale = w_scale;
  p.bias = static_cast<const __nv_bfloat16*>(bias);
  p.out = out;
  p.epi = epi;
  p.err = device_error_flag();
  const int tiles = p.m_blocks * p.n_blocks;
  const int grid = tiles < sm_count() ? tiles : sm_count();
  // The gated residual and the fp32 store (the patchify projection, whose epilogue is
  // nearly all of its time) take the staged epilogue.
  const bool staged = epi.kind == WAN_EPI_RESIDUAL || epi.kind == WAN_EPI_F32;
  return staged ? launch_inst<BN, kF8, true>(mapA, mapB, p, grid, s) : launch_inst<BN, kF8, false>(mapA, mapB, p, grid, s);
}

}  // namespace

int launch_gemm_tc(const void* A, int64_t lda, const void* W, const void* bias, void* out, int M, int N, int K,
                   int w_k_period, const GemmEpi& epi, cudaStream_t s) {
  if (M == 0 || N == 0) return WAN_OK;
  if (K % 8 != 0 || lda % 8 != 0 || N % 8 != 0) return WAN_ERR_SHAPE;
  if (w_k_period > 0 && (w_k_period % kBK != 0 || K % w_k_period != 0)) return WAN_ERR_SHAPE;
  trace_launch_begin(WAN_KIND_GEMM, s, 2.0 * M * N * K);
  int st;
  if (N <= 64)
    st = launch_bn<64, false>(A, lda, W, bias, out, M, N, K, w_k_period, epi, s);
  else if (N <= 128)
    st = launch_bn<128, false>(A, lda, W, bias, out, M, N, K, w_k_period, epi, s);
  else if (WAN_GEMM_PAIR && N >= 256 && K >= 256 && M >= 1024 && sm_count() >= 2)
    // long enough main loops and enough row blocks for the pair tiles to pay (the patchify
    // projection, K = 64, and the 512-row context projections stay on one SM)
    st = launch_pair<false>(A, lda, W, bias, out, M, N, K, w_k_period, epi, s);
  else
    st = launch_bn<256, false>(A, lda, W, bias, out, M, N, K, w_k_period, epi, s);
  trace_launch_end(WAN_KIND_GEMM, s);
  return st;
}

int launch_gemm_e4m3(const void* A, int64_t lda, const float* a_scale, const void* W, const float* w_scale,
                     const void* bias, void* out, int M, int N, int K, const GemmEpi& epi, cudaStream_t s) {
  if (M == 0 || N == 0) return WAN_OK;
  if (K % 16 != 0 || lda % 16 != 0 || N % 8 != 0) return WAN_ERR_SHAPE;
  trace_launch_begin(WAN_KIND_GEMM, s, 2.0 * M * N * K);
  int st;
  if (N <= 64)
    st = launch_bn<64, true>(A, lda, W, bias, out, M, N, K, 0, epi, s, a_scale, w_scale);
  else if (N <= 128)
    st = launch_bn<128, true>(A, lda, W, bias, out, M, N, K, 0, epi, s, a_scale, w_scale);
  else if (WAN_GEMM_PAIR && N >= 256 && K >= 512 && M >= 1024 && sm_count() >= 2)
    st = launch_pair<true>(A, lda, W, bias, out, M, N, K, 0, epi, s, a_scale, w_scale);
  else
    st = launch_bn<256, true>(A, lda, W, bias, out, M, N, K, 0, epi, s, a_scale, w_scale);
  trace_launch_end(WAN_KIND_GEMM, s);
  return st;
}

}  // namespace wan
