// Kernel (b): flash-attention forward on the sm_100a tensor cores for the Wan 2.1 DiT
// ("Wan: Open and Advanced Large-Scale Video Generative Models", section "Diffusion
// Transformer": full spatio-temporal self-attention over all L video tokens, and text
// cross-attention over 512 umT5 tokens in every block). softmax(q k^T / sqrt(d)) v per
// head, non-causal, bf16 inputs, fp32 accumulation and fp32 softmax, head_dim 128.
//
// One CTA = two 128-row query tiles (t = 0, 1) of one (sample, head); 384 threads in
// three warpgroups (bf16; the E4M3 instantiation has 320 threads, no idle warps, and
// its softmax warps are 2-5 and 6-9):
//   warp 0    : TMA producer - both Q tiles once, then K_0, K_1, V_0, K_2, V_1, ...
//               (the order the MMA warp consumes them) through a 5-stage ring of 32 KB
//               tiles (128 rows x 128 dims as two 64-dim halves, 128-byte swizzle);
//   warp 1    : one thread issues tcgen05.mma. For key tile j and each query tile t:
//               O_t += P_t(j-1) V_{j-1} (P read from tensor memory, V an MN-major
//               operand in shared memory), then S_t = Q_t K_j^T, then a commit that
//               signals S_t ready. MMAs of one thread execute in issue order, so that
//               signal also means P_t has been consumed and O_t holds every earlier PV;
//   warps 2-3 : idle (they complete warpgroup 0, which hands registers to the softmax);
//   warps 4-7 : softmax of query tile 0, warps 8-11: of query tile 1; one thread per
//               query row (warp % 4 selects the TMEM lane quarter). The row's 128 S
//               values are read from TMEM with a single wait (the wait covers every
//               outstanding TMEM load, so reading in pieces would expose its latency
//               once per piece); fp32 max and sum, ex2, the ragged last key tile
//               masked only on that tile. Scaling and row sums run on packed f32x2
//               pairs (one instruction per pair), which leaves more issue slots to the
//               other tile's softmax warp and the MMA warp on the same SM sub-partition. P is rounded to bf16, packed in place and
//               written back into tensor memory over the S columns already read (two
//               bf16 per 32-bit column, the layout of a K-major MMA operand), so P
//               never touches shared memory.
//               The exponent base moves only when the row max grows by more than 2^8
//               (O_t in TMEM and the sum are rescaled then): softmax is invariant to the
//               base and p <= 256 stays well inside fp32 and bf16 range.
// While one tile's softmax runs, the tensor core works on the other tile's MMAs.
// Registers (bf16): the CTA launches at 168 a thread (the most 384 threads may hold);
// then warpgroup 0 gives up all but 88 (setmaxnreg.dec) and the two softmax warpgroups
// take 208 (setmaxnreg.inc): 128 x 88 + 256 x 208 = 384 x 168, and on each SM
// sub-partition (one warp of each warpgroup) 88 + 208 + 208 = 3 x 168, so every increase
// is covered by the decrease. The softmax keeps a whole 128-value S row in registers; at
// 168 a thread it spilled loop state. The E4M3 kernel did not spill at 168 and measured
// about 1 % slower with the split, so it keeps 320 threads at 168.
// Work units are (sample, head, pair of query tiles), one CTA each, in a 1D grid. When
// the last wave would fill at most half of the SMs, its units are split over the key
// tiles instead (two CTAs per unit, each over half of them); those CTAs write their
// unnormalised output with each row's base and sum to a caller scratch, and
// attn_combine_kernel merges the halves.
// TMEM: S_0 (later P_0), S_1 (P_1), O_0, O_1 = 4 x 128 of the 512 columns.
//
// The E4M3 instantiation (kF8; the 8-bit attention of the same page's section "Infra",
// inference optimisation, here with E4M3 for both products) runs the same protocol on
// E4M3 codes: 16 KB tiles (128 codes per 128-byte swizzled row), an 8-stage ring, four
// kind::f8f6f4 MMAs of K = 32 per product, P as four E4M3 codes per TMEM column, and V
// stored transposed so that both products take K-major operands. A row's q scale and
// its head's k scale fold into the row's log2 scale, the v scale into the output. The
// running base is rounded up to a whole power of two, so that P's codes equal those of
// the final base times an exact power of two (outside E4M3's subnormal range) and every
// rescale factor is exact. With the products at twice the rate the exponentials are the
// busier unit, so one in eight runs on the FMA pipes (exp2_poly).
#include <cuda_bf16.h>

#include <math.h>

#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace wan {
namespace {

constexpr int kRegsLow = 88;    // warpgroup 0 (producer, MMA issuer, two idle warps)
constexpr int kRegsHigh = 208;  // warpgroups 1-2 (softmax)
static_assert(128 * kRegsLow + 256 * kRegsHigh <= 384 * 168, "register split above the launch");
static_assert(kRegsLow + 2 * kRegsHigh <= 3 * 168, "register split above a sub-partition's share");
constexpr int kTile = 128;                     // query rows per tile = key rows per tile
constexpr int kHd = 128;                       // head dim
constexpr int kQTiles = 2;                     // query tiles per CTA
constexpr int kHalfBytes = kTile * 128;        // 128 rows of one 128-byte swizzled span

// Operand shapes: bf16 tiles are two 64-column spans (32 KB), E4M3 tiles one span of
// 128 codes (16 KB). K of one MMA is 16 (bf16) or 32 (E4M3), so a 128-deep product
// takes 8 or 4 instructions. The 16 KB tiles leave room for a deeper K/V ring.
// The persistent variant (kPersist, short key sequences) double-buffers Q so that the
// next unit's Q lands while the current one computes; its K/V ring is 3 stages to fit.
template <bool kF8, bool kPersist = false>
struct AttnShape {
  static constexpr int kTileBytes = kTile * (kF8 ? 128 : 256);
  static constexpr int kSpans = kF8 ? 1 : 2;
  static constexpr int kQBufs = kPersist ? 2 : 1;
  static constexpr int kStages = kPersist ? 3 : (kF8 ? 8 : 5);
  static constexpr int kMmas = kF8 ? 4 : 8;
  // bf16: three warpgroups with the register split; E4M3: 320 threads, no split
  static constexpr bool kRegSplit = !kF8;
  static constexpr int kThreads = kRegSplit ? 384 : 320;
  static constexpr int kSoftmaxWarp0 = kRegSplit ? 4 : 2;  // first softmax warp
  static constexpr size_t kSmem =
      1024 + static_cast<size_t>(kTileBytes) * (kQBufs * kQTiles + kStages) + 256;
};
// Key sequences of at most this many 128-key tiles (the 512 text and 257 image tokens of
// the cross-attention) run on the persistent variant.
constexpr int kMaxPersistKeyTiles = 4;
constexpr float kRescaleLog2 = 8.0f;
constexpr int kMinSplitKeyTiles = 16;          // see launch_attn_tc

struct AttnParams {
  int Lq, Lk, H;
  int q_col0, k_col0, v_col0;
  float scale_log2;  // log2(e) / sqrt(d)
  __nv_bfloat16* o;
  int64_t o_row_stride;
  int64_t o_batch_stride;
  int o_col0;
  SeqScatter sc;  // sc.ranks > 0: rows go to their owners' buffers
  // Work units: (sample, head, pair of query tiles), unit = (b * H + h) * pairs + pair.
  // CTAs [0, n_full) take one unit over all key tiles; the CTAs after them split the
  // remaining units' key tiles in two halves (CTA n_full + 2u + half) and write
  // unnormalised partial outputs to part_o / part_ml, merged by attn_combine_kernel.
  int pairs, n_full;
  int n_units;     // persistent variant: CTA c takes units c, c + gridDim.x, ...
  float* part_o;   // [split CTA][tile][128 rows][128] fp32
  float* part_ml;  // [split CTA][tile][128 rows][2] (row max, row sum) fp32
  // E4M3 operands only: q scale per (sample, query row, head) [B, Lq, H]; k and v scale
  // per (sample, head) [B, H, 2]. V is stored transposed ([B, H*128 dims, keys]).
  const float* q_scale;
  const float* kv_scale;
  int* err;
};

// Ring position of K_j / V_j in the load order K_0, K_1, V_0, K_2, V_1, ..., V_{n-1}.
__device__ __forceinline__ int pos_k(int j) { return j == 0 ? 0 : 2 * j - 1; }
__device__ __forceinline__ int pos_v(int j, int n) { return j == n - 1 ? 2 * n - 1 : 2 * j + 2; }

template <bool kF8, bool kPersist>
__global__ void __launch_bounds__(AttnShape<kF8, kPersist>::kThreads, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                       const __grid_constant__ CUtensorMap mapV, const AttnParams p) {
  using Shape = AttnShape<kF8, kPersist>;
  constexpr int kTileBytes = Shape::kTileBytes;
  constexpr int kStages = Shape::kStages;
  constexpr int kSpans = Shape::kSpans;
  constexpr int kMmas = Shape::kMmas;
  constexpr int kQBufs = Shape::kQBufs;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                                  // [kQBufs][2][tile]
  uint8_t* sKV = sQ + kQBufs * kQTiles * kTileBytes;   // [kStages][tile]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + kStages * kTileBytes);
  uint64_t* q_full = bars;                 // [kQBufs]
  uint64_t* q_empty = q_full + kQBufs;     // [kQBufs] (persistent: Q buffer free again)
  uint64_t* kv_full = q_empty + kQBufs;
  uint64_t* kv_empty = kv_full + kStages;
  uint64_t* s_full = kv_empty + kStages;   // [2]
  uint64_t* p_full = s_full + kQTiles;     // [2]
  uint64_t* o_final = p_full + kQTiles;    // [2]
  uint64_t* drain = o_final + kQTiles;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nkv_all = (p.Lk + kTile - 1) / kTile;
  // Work of this CTA: one unit (possibly one key half of a split unit), or, persistent,
  // units blockIdx.x, blockIdx.x + gridDim.x, ... over all key tiles. Every barrier
  // phase below counts across the units a CTA takes: Q buffer fills per buffer, ring
  // loads, key tiles (S ready / P ready) and units (O final).
  int kv0 = 0, kv1 = nkv_all, split = -1;
  int n_iter = 1;
  if constexpr (kPersist) {
    n_iter = blockIdx.x < p.n_units ? (p.n_units - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                                    : 0;
  } else if (static_cast<int>(blockIdx.x) >= p.n_full) {
    split = blockIdx.x - p.n_full;
    kv0 = (split & 1) ? nkv_all / 2 : 0;
    kv1 = (split & 1) ? nkv_all : nkv_all / 2;
  }
  const int nkv = kv1 - kv0;  // key tiles this CTA visits per unit, from key tile kv0 on
  auto unit_of = [&](int it) {
    if constexpr (kPersist) return static_cast<int>(blockIdx.x) + it * static_cast<int>(gridDim.x);
    return split >= 0 ? p.n_full + (split >> 1) : static_cast<int>(blockIdx.x);
  };
  struct UnitPos {
    int b, h, q0;
  };
  auto decode = [&](int unit) {
    const int bh = unit / p.pairs;
    return UnitPos{bh / p.H, bh % p.H, (unit - bh * p.pairs) * (kQTiles * kTile)};
  };

  if (threadIdx.x == 0) {
    for (int q = 0; q < kQBufs; ++q) {
      mbar_init(&q_full[q], 1);
      mbar_init(&q_empty[q], 1);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int t = 0; t < kQTiles; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 128);
      mbar_init(&o_final[t], 1);
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

  if (warp < Shape::kSoftmaxWarp0) {
    if constexpr (Shape::kRegSplit) setmaxnreg_dec<kRegsLow>();
    if (warp == 0) {
      if (lane == 0) {
        const int n_loads = 2 * nkv;
        int issued = 0;  // ring loads issued so far (all units)
        int q_loads = 0;
        bool ok = true;
        for (int it = 0; ok && it < n_iter; ++it) {
          const UnitPos u = decode(unit_of(it));
          const int qb = it % kQBufs;
          if (kPersist && it >= kQBufs &&
              !mbar_wait(&q_empty[qb], static_cast<uint32_t>((it / kQBufs - 1) & 1), p.err))
            break;
          uint8_t* sq = sQ + qb * kQTiles * kTileBytes;
          mbar_arrive_expect_tx(&q_full[qb], kQTiles * kTileBytes);
          const int qc = p.q_col0 + u.h * kHd;
          for (int t = 0; t < kQTiles; ++t)
            for (int c = 0; c < kSpans; ++c)
              tma_load_3d(sq + t * kTileBytes + c * kHalfBytes, &mapQ, &q_full[qb], qc + 64 * c, u.q0 + t * kTile, u.b);
          ++q_loads;
          for (int ld = 0; ld < n_loads; ++ld) {
            const int stage = issued % kStages;
            const uint32_t phase = static_cast<uint32_t>((issued / kStages) & 1);
            if (!mbar_wait(&kv_empty[stage], phase ^ 1u, p.err)) {
              ok = false;
              break;
            }
            bool is_v;
            int j;
            if (ld == 0) {
              is_v = false, j = 0;
            } else if (ld == n_loads - 1) {
              is_v = true, j = nkv - 1;
            } else if (ld & 1) {
              is_v = false, j = (ld + 1) >> 1;
            } else {
              is_v = true, j = (ld >> 1) - 1;
            }
            const CUtensorMap* map = is_v ? &mapV : &mapK;
            const int col = (is_v ? p.v_col0 : p.k_col0) + u.h * kHd;
            uint8_t* dst = sKV + stage * kTileBytes;
            mbar_arrive_expect_tx(&kv_full[stage], kTileBytes);
            if (kF8 && is_v) {  // V^T: 128 dims (rows) x 128 keys (x)
              tma_load_3d(dst, map, &kv_full[stage], (kv0 + j) * kTile, p.v_col0 + u.h * kHd, u.b);
            } else {
              for (int c = 0; c < kSpans; ++c)
                tma_load_3d(dst + c * kHalfBytes, map, &kv_full[stage], col + 64 * c, (kv0 + j) * kTile, u.b);
            }
            ++issued;
          }
        }
        // Wait for every copy this thread started (the last fill of each buffer and stage).
        for (int q = 0; q < kQBufs; ++q) {
          const int n_q = q_loads / kQBufs + (q < q_loads % kQBufs ? 1 : 0);
          if (n_q > 0) mbar_wait(&q_full[q], static_cast<uint32_t>((n_q - 1) & 1), p.err);
        }
        for (int s = 0; s < kStages; ++s) {
          const int n_s = issued / kStages + (s < issued % kStages ? 1 : 0);
          if (n_s > 0) mbar_wait(&kv_full[s], static_cast<uint32_t>((n_s - 1) & 1), p.err);
        }
      }
    } else if (warp == 1) {
      if (lane == 0) {
        const uint32_t idesc_qk = kF8 ? idesc_e4m3_f32(kTile, kTile) : idesc_bf16_f32(kTile, kTile, 0, 0);
        // PV: bf16 V is an MN-major operand; E4M3 V arrives transposed, so K-major.
        const uint32_t idesc_pv = kF8 ? idesc_e4m3_f32(kTile, kHd) : idesc_bf16_f32(kTile, kHd, 0, 1);
        // Shared-memory descriptors are built once: every operand below sits at a fixed
        // byte offset from sQ or sKV, and an offset moves only the 14-bit address field
        // (offset >> 4, no carry out of it since shared addresses stay below 256 KB). The
        // single issuing thread then spends one add per operand on each MMA.
        const uint64_t q_desc = sdesc_sw128(smem_u32(sQ), 16, 1024);
        const uint64_t k_desc = sdesc_sw128(smem_u32(sKV), 16, 1024);
        const uint64_t v_desc = sdesc_sw128(smem_u32(sKV), kF8 ? 16 : kHalfBytes, 1024);
        auto wait_pos = [&](int pos) {
          return mbar_wait(&kv_full[pos % kStages], static_cast<uint32_t>((pos / kStages) & 1), p.err);
        };
        auto pv = [&](int t, int i, int vstage) {
          // A = P_t in TMEM, packed from the first column of S_t's region (bf16 pairs or
          // E4M3 quads per column, so 8 columns per MMA either way).
          const uint32_t p_tmem = tmem_base + t * kTile;
          const uint64_t vd = v_desc + static_cast<uint32_t>((vstage * kTileBytes) >> 4);
          const uint32_t o_tmem = tmem_base + 256 + t * kTile;
#pragma unroll
          for (int k = 0; k < kMmas; ++k) {
            const uint32_t acc = (i > 0 || k > 0) ? 1u : 0u;
            if constexpr (kF8)
              tc_mma_e4m3_ts(o_tmem, p_tmem + k * 8, vd + ((k * 32) >> 4), idesc_pv, acc);
            else
              tc_mma_bf16_ts(o_tmem, p_tmem + k * 8, vd + ((k * 16 * 128) >> 4), idesc_pv, acc);
          }
        };
        auto qk = [&](int t, int qb, int kstage) {
          const uint64_t qd = q_desc + static_cast<uint32_t>(((qb * kQTiles + t) * kTileBytes) >> 4);
          const uint64_t kd = k_desc + static_cast<uint32_t>((kstage * kTileBytes) >> 4);
          const uint32_t s_tmem = tmem_base + t * kTile;
#pragma unroll
          for (int k = 0; k < kMmas; ++k) {
            const uint32_t off = ((k >> 2) * kHalfBytes + (k & 3) * 32) >> 4;  // 32 bytes of K per MMA
            if constexpr (kF8)
              tc_mma_e4m3(s_tmem, qd + off, kd + off, idesc_qk, k > 0 ? 1u : 0u);
            else
              tc_mma_bf16(s_tmem, qd + off, kd + off, idesc_qk, k > 0 ? 1u : 0u);
          }
        };
        bool ok = true;
        for (int it = 0; ok && it < n_iter; ++it) {
          const int qb = it % kQBufs;
          const int base = it * 2 * nkv;   // ring position of this unit's first load
          const int tiles = it * nkv;      // key tiles of earlier units (S / P phases)
          if (!mbar_wait(&q_full[qb], static_cast<uint32_t>((it / kQBufs) & 1), p.err)) break;
          for (int j = 0; ok && j < nkv; ++j) {
            const int pk = base + pos_k(j);
            if (!wait_pos(pk)) {
              ok = false;
              break;
            }
            int pvpos = -1;
            if (j > 0) {
              pvpos = base + pos_v(j - 1, nkv);
              if (!wait_pos(pvpos)) {
                ok = false;
                break;
              }
            }
            for (int t = 0; ok && t < kQTiles; ++t) {
              if (j > 0) {
                if (!mbar_wait(&p_full[t], static_cast<uint32_t>((tiles + j - 1) & 1), p.err)) {
                  ok = false;
                  break;
                }
                // The first PV of a unit overwrites O_t. The softmax threads of tile t
                // read the previous unit's O_t out (and waited for those reads) before
                // they arrived on p_full for this unit's first key tile, so it is free.
                tc_fence_after();
                pv(t, j - 1, pvpos % kStages);
              }
              qk(t, qb, pk % kStages);
              tc_commit(&s_full[t]);
            }
            if (!ok) break;
            tc_commit(&kv_empty[pk % kStages]);
            if (j > 0) tc_commit(&kv_empty[pvpos % kStages]);
          }
          if (!ok || nkv == 0) break;
          tc_commit(&q_empty[qb]);   // every QK of this unit issued: Q buffer free once they complete
          const int last = nkv - 1;
          const int pvpos = base + pos_v(last, nkv);
          ok = wait_pos(pvpos);
          for (int t = 0; ok && t < kQTiles; ++t) {
            if (!mbar_wait(&p_full[t], static_cast<uint32_t>((tiles + last) & 1), p.err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            pv(t, last, pvpos % kStages);
            tc_commit(&o_final[t]);
          }
          if (!ok) break;
          tc_commit(&kv_empty[pvpos % kStages]);
        }
        tc_commit(drain);
        mbar_wait(drain, 0, p.err);
      }
    }
  } else {
    if constexpr (Shape::kRegSplit) setmaxnreg_inc<kRegsHigh>();
    // Softmax: query tile t, TMEM lane quarter (warp % 4), row 32 * quarter + lane.
    const int t = (warp - Shape::kSoftmaxWarp0) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t s_row = tmem_base + lane_off + t * kTile;
    const uint32_t o_row = tmem_base + lane_off + 256 + t * kTile;
    bool ok = true;
    for (int it = 0; ok && it < n_iter; ++it) {
      const UnitPos u = decode(unit_of(it));
      const int b = u.b, h = u.h, q0 = u.q0;
      const int tiles = it * nkv;
      float sl2 = p.scale_log2;
      float v_scale = 1.0f;
      if constexpr (kF8) {
        // Logit = S q_scale k_scale / sqrt(d): the row's scales fold into its log2 scale;
        // the v scale multiplies the output.
        const float* kvs = p.kv_scale + 2 * (static_cast<int64_t>(b) * p.H + h);
        const int grow0 = q0 + t * kTile + row;
        sl2 *= kvs[0] * (grow0 < p.Lq ? p.q_scale[(static_cast<int64_t>(b) * p.Lq + grow0) * p.H + h] : 1.0f);
        v_scale = kvs[1];
      }
      float m_run = -INFINITY;
      float l_run = 0.f;
      for (int j = 0; ok && j < nkv; ++j) {
        if (!mbar_wait_warp(&s_full[t], static_cast<uint32_t>((tiles + j) & 1), p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int valid = p.Lk - (kv0 + j) * kTile;  // keys of this tile that exist (mask the rest)
        // The whole S row (128 fp32) is read with one wait; P is then packed in place into
        // the first 64 registers (pair i of the row lands in register i <= 2i, so the pass
        // never overwrites a value it still has to read) and stored over S in TMEM.
        uint32_t r[kTile];
        tmem_ld32(s_row, *reinterpret_cast<uint32_t(*)[32]>(r));
        tmem_ld32(s_row + 32, *reinterpret_cast<uint32_t(*)[32]>(r + 32));
        tmem_ld32(s_row + 64, *reinterpret_cast<uint32_t(*)[32]>(r + 64));
        tmem_ld32(s_row + 96, *reinterpret_cast<uint32_t(*)[32]>(r + 96));
        tmem_ld_wait();
        if (valid < kTile) {
#pragma unroll
          for (int i = 0; i < kTile; ++i)
            if (i >= valid) r[i] = __float_as_uint(-INFINITY);
        }
        float mx8[8];
#pragma unroll
        for (int a = 0; a < 8; ++a) mx8[a] = __uint_as_float(r[a]);
#pragma unroll
        for (int i = 8; i < kTile; i += 2)
          mx8[(i >> 1) & 7] = fmax3(mx8[(i >> 1) & 7], __uint_as_float(r[i]), __uint_as_float(r[i + 1]));
        const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                               fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        const bool grow = (mx - m_run) * sl2 > kRescaleLog2;
        float alpha = 1.0f;
        bool rescale = false;
        if (j == 0) {
          m_run = mx;
        } else if (__any_sync(0xffffffffu, grow)) {
          const float m_new = fmaxf(m_run, mx);
          // E4M3 P: bases are whole powers of two (see below), so alpha is one as well.
          alpha = kF8 ? pow2i(static_cast<int>(ceilf(m_run * sl2) - ceilf(m_new * sl2)))
                      : ex2_approx((m_run - m_new) * sl2);
          m_run = m_new;
          rescale = true;
        }
        // E4M3 P is taken against the base rounded up to a whole power of two: p <= 2^8
        // still, and its codes are those of the exact-max base times an exact power of two
        // (outside the subnormal range), whatever this row's running max is.
        const float nb = kF8 ? -ceilf(m_run * sl2) : -m_run * sl2;
        const unsigned long long sl2x2 = f2_pack(sl2, sl2), nbx2 = f2_pack(nb, nb);
        unsigned long long rs4[4] = {0ull, 0ull, 0ull, 0ull};
        if constexpr (kF8) {
          // E4M3 P: four codes per register (quad i of the row lands in register i <= 4i).
#pragma unroll
          for (int i = 0; i < kTile / 4; ++i) {
            const unsigned long long s01 = f2_pack(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]));
            const unsigned long long s23 = f2_pack(__uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
            const float2 x01 = f2_unpack(f2_fma(s01, sl2x2, nbx2));
            const float2 x23 = f2_unpack(f2_fma(s23, sl2x2, nbx2));
            const float e0 = ex2_approx(x01.x), e1 = ex2_approx(x01.y);
            // one exponential in eight on the FMA pipes (MUFU is the busier unit here)
            const float e2 = ex2_approx(x23.x);
            const float e3 = (i & 1) == 0 ? exp2_poly(x23.y) : ex2_approx(x23.y);
            rs4[(2 * i) & 3] = f2_add(rs4[(2 * i) & 3], f2_pack(e0, e1));
            rs4[(2 * i + 1) & 3] = f2_add(rs4[(2 * i + 1) & 3], f2_pack(e2, e3));
            r[i] = pack_e4m3x4(e0, e1, e2, e3);
          }
          tmem_st32(s_row, *reinterpret_cast<uint32_t(*)[32]>(r));
        } else {
#pragma unroll
          for (int i = 0; i < kTile / 2; ++i) {
            const unsigned long long s2 = f2_pack(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
            const float2 x = f2_unpack(f2_fma(s2, sl2x2, nbx2));
            const float e0 = ex2_approx(x.x);
            const float e1 = ex2_approx(x.y);
            rs4[i & 3] = f2_add(rs4[i & 3], f2_pack(e0, e1));
            r[i] = pack_bf16x2(e0, e1);
          }
          tmem_st32(s_row, *reinterpret_cast<uint32_t(*)[32]>(r));
          tmem_st32(s_row + 32, *reinterpret_cast<uint32_t(*)[32]>(r + 32));
        }
        if (rescale) {
          // S_t(j) ready implies PV_t(j-1) completed, and PV_t(j) waits for this thread's
          // arrival below: O_t is current and idle while it is rescaled here.
#pragma unroll 1
          for (int c = 0; c < kHd / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(o_row + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 32; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha);
            tmem_st32(o_row + c * 32, o);
          }
          l_run *= alpha;
        }
        {
          const float2 s01 = f2_unpack(f2_add(rs4[0], rs4[1])), s23 = f2_unpack(f2_add(rs4[2], rs4[3]));
          l_run += (s01.x + s01.y) + (s23.x + s23.y);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[t]);
      }
      const bool done = ok && nkv > 0 && mbar_wait_warp(&o_final[t], static_cast<uint32_t>(it & 1), p.err);
      if (!done) ok = false;
      if (done && split >= 0) {
        // Partial output of a key-split CTA: O unnormalised, with the row's base and sum.
        tc_fence_after();
        const int64_t slot = (static_cast<int64_t>(split) * kQTiles + t) * kTile + row;
        float4* po = reinterpret_cast<float4*>(p.part_o + slot * kHd);
#pragma unroll 1
        for (int c = 0; c < kHd / 32; ++c) {
          uint32_t r0[32];
          tmem_ld32(o_row + c * 32, r0);
          tmem_ld_wait();
#pragma unroll
          for (int g = 0; g < 8; ++g)
            po[c * 8 + g] = make_float4(__uint_as_float(r0[4 * g]), __uint_as_float(r0[4 * g + 1]),
                                        __uint_as_float(r0[4 * g + 2]), __uint_as_float(r0[4 * g + 3]));
        }
        // E4M3: the whole-power-of-two base itself (the merge then uses scale 1).
        const float m_common = kF8 ? ceilf(m_run * sl2) : m_run;
        reinterpret_cast<float2*>(p.part_ml)[slot] = make_float2(m_common, l_run);
      } else if (done) {
        tc_fence_after();
        const float inv = v_scale / l_run;
        const int grow = q0 + t * kTile + row;
        __nv_bfloat16* orow;
        if (p.sc.ranks > 0) {
          const int owner = min(grow / p.sc.rows_local, p.sc.ranks - 1);
          const int64_t lrow = static_cast<int64_t>(b) * p.sc.rows_local + (grow - owner * p.sc.rows_local);
          orow = static_cast<__nv_bfloat16*>(p.sc.dst[owner]) + lrow * p.o_row_stride + p.o_col0 + h * kHd;
        } else {
          orow = p.o + static_cast<int64_t>(b) * p.o_batch_stride + static_cast<int64_t>(grow) * p.o_row_stride +
                 p.o_col0 + h * kHd;
        }
#pragma unroll
        for (int c = 0; c < kHd / 64; ++c) {
          uint32_t r0[32], r1[32];
          tmem_ld32(o_row + c * 64, r0);
          tmem_ld32(o_row + c * 64 + 32, r1);
          tmem_ld_wait();
          if (grow < p.Lq) {
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              uint4 u4;
              u4.x = pack_bf16x2(__uint_as_float(r0[g * 8 + 0]) * inv, __uint_as_float(r0[g * 8 + 1]) * inv);
              u4.y = pack_bf16x2(__uint_as_float(r0[g * 8 + 2]) * inv, __uint_as_float(r0[g * 8 + 3]) * inv);
              u4.z = pack_bf16x2(__uint_as_float(r0[g * 8 + 4]) * inv, __uint_as_float(r0[g * 8 + 5]) * inv);
              u4.w = pack_bf16x2(__uint_as_float(r0[g * 8 + 6]) * inv, __uint_as_float(r0[g * 8 + 7]) * inv);
              reinterpret_cast<uint4*>(orow + c * 64)[g] = u4;
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(r1[g * 8 + 0]) * inv, __uint_as_float(r1[g * 8 + 1]) * inv);
              w.y = pack_bf16x2(__uint_as_float(r1[g * 8 + 2]) * inv, __uint_as_float(r1[g * 8 + 3]) * inv);
              w.z = pack_bf16x2(__uint_as_float(r1[g * 8 + 4]) * inv, __uint_as_float(r1[g * 8 + 5]) * inv);
              w.w = pack_bf16x2(__uint_as_float(r1[g * 8 + 6]) * inv, __uint_as_float(r1[g * 8 + 7]) * inv);
              reinterpret_cast<uint4*>(orow + c * 64 + 32)[g] = w;
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

// Merge the two key halves of each split unit: with m = max(m0, m1) and
// w_i = 2^((m_i - m) scale_log2), O = (w0 O0 + w1 O1) / (w0 l0 + w1 l1). One block per
// (split unit, query tile); each warp takes rows, each lane 4 of the 128 columns.
__global__ void __launch_bounds__(256) attn_combine_kernel(const AttnParams p) {
  const int u = blockIdx.x, t = blockIdx.y;
  const int unit = p.n_full + u;
  const int bh = unit / p.pairs;
  const int q0 = (unit - bh * p.pairs) * (kQTiles * kTile) + t * kTile;
  const int h = bh % p.H, b = bh / p.H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int r = warp; r < kTile; r += 8) {
    const int grow = q0 + r;
    if (grow >= p.Lq) break;
    const int64_t s0 = (static_cast<int64_t>(2 * u) * kQTiles + t) * kTile + r;
    const int64_t s1 = (static_cast<int64_t>(2 * u + 1) * kQTiles + t) * kTile + r;
    const float2 ml0 = reinterpret_cast<const float2*>(p.part_ml)[s0];
    const float2 ml1 = reinterpret_cast<const float2*>(p.part_ml)[s1];
    const float m = fmaxf(ml0.x, ml1.x);
    const float ms = p.kv_scale ? 1.0f : p.scale_log2;  // E4M3 partials carry log2 bases
    const float w0 = exp2f((ml0.x - m) * ms), w1 = exp2f((ml1.x - m) * ms);
    const float v_scale = p.kv_scale ? p.kv_scale[2 * (static_cast<int64_t>(b) * p.H + h) + 1] : 1.0f;
    const float inv = v_scale / (w0 * ml0.y + w1 * ml1.y);
    const float4 a = reinterpret_cast<const float4*>(p.part_o + s0 * kHd)[lane];
    const float4 c = reinterpret_cast<const float4*>(p.part_o + s1 * kHd)[lane];
    uint2 v;
    v.x = pack_bf16x2((w0 * a.x + w1 * c.x) * inv, (w0 * a.y + w1 * c.y) * inv);
    v.y = pack_bf16x2((w0 * a.z + w1 * c.z) * inv, (w0 * a.w + w1 * c.w) * inv);
    __nv_bfloat16* orow = p.o + static_cast<int64_t>(b) * p.o_batch_stride + static_cast<int64_t>(grow) * p.o_row_stride +
                          p.o_col0 + h * kHd;
    reinterpret_cast<uint2*>(orow)[lane] = v;
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

template <bool kF8, bool kPersist>
void set_attn_smem_once(int dev) {
  static std::once_flag once[64];
  std::call_once(once[dev & 63], [] {
    cudaFuncSetAttribute(attn_fwd_tc_kernel<kF8, kPersist>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(AttnShape<kF8, kPersist>::kSmem));
  });
}

// Grid, optional key split of a partial last wave, launch and merge (both operand kinds).
template <bool kF8>
int launch_units(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, AttnParams& p, int B, int H,
                 int Lq, int Lk, cudaStream_t s, bool has_sc, void* scratch, size_t scratch_bytes) {
  p.err = device_error_flag();
  int dev = 0;
  cudaGetDevice(&dev);
  p.pairs = (Lq + kQTiles * kTile - 1) / (kQTiles * kTile);
  const int64_t units = static_cast<int64_t>(B) * H * p.pairs;
  if (units >= (int64_t(1) << 31)) return WAN_ERR_SHAPE;
  p.n_units = static_cast<int>(units);
  static int nsm_of[64] = {0};
  if (nsm_of[dev & 63] == 0) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    nsm_of[dev & 63] = v > 0 ? v : 148;
  }
  const int nsm = nsm_of[dev & 63];
  const int nkv_all = (Lk + kTile - 1) / kTile;
  const double work = 4.0 * B * H * static_cast<double>(Lq) * Lk * kHd;
  // Short key sequences (a unit is a few key tiles long, so loading Q, setting up and
  // writing O would dominate a one-unit CTA): one persistent CTA per SM walks the
  // units, loading the next unit's Q and starting its first products while the
  // current unit's output is written.
  if (!kF8 && nkv_all <= kMaxPersistKeyTiles) {
    set_attn_smem_once<kF8, true>(dev);
    p.n_full = p.n_units;
    p.part_o = p.part_ml = nullptr;
    const unsigned grid = static_cast<unsigned>(units < nsm ? units : nsm);
    trace_launch_begin(WAN_KIND_ATTN, s, work);
    attn_fwd_tc_kernel<kF8, true>
        <<<grid, AttnShape<kF8, true>::kThreads, AttnShape<kF8, true>::kSmem, s>>>(mq, mk, mv, p);
    const int st = check_launch();
    trace_launch_end(WAN_KIND_ATTN, s);
    return st;
  }
  set_attn_smem_once<kF8, false>(dev);
  constexpr size_t kSmem = AttnShape<kF8>::kSmem;
  // One CTA per unit. When the last wave would leave more than half of the SMs idle,
  // its units are split over the key tiles instead (two CTAs each) and merged after.
  const int64_t rem = units % nsm;
  const size_t part_o_bytes = static_cast<size_t>(2 * rem) * kQTiles * kTile * kHd * 4;
  const size_t part_bytes = part_o_bytes + static_cast<size_t>(2 * rem) * kQTiles * kTile * 8;
  // Only when a unit is long enough (16+ key tiles) for half of it to outweigh the
  // partial-output traffic and the merge launch (at 4 key tiles, as in the text
  // cross-attention, splitting measured 9 % slower).
  const bool split = rem > 0 && 2 * rem <= nsm && nkv_all >= kMinSplitKeyTiles && !has_sc && scratch &&
                     scratch_bytes >= part_bytes && (reinterpret_cast<uintptr_t>(scratch) & 15u) == 0;
  p.n_full = static_cast<int>(split ? units - rem : units);
  p.part_o = split ? static_cast<float*>(scratch) : nullptr;
  p.part_ml = split ? reinterpret_cast<float*>(static_cast<uint8_t*>(scratch) + part_o_bytes) : nullptr;
  const unsigned grid = static_cast<unsigned>(split ? units + rem : units);
  trace_launch_begin(WAN_KIND_ATTN, s, work);
  attn_fwd_tc_kernel<kF8, false><<<grid, AttnShape<kF8, false>::kThreads, kSmem, s>>>(mq, mk, mv, p);
  int st = check_launch();
  if (st == WAN_OK && split) {
    attn_combine_kernel<<<dim3(static_cast<unsigned>(rem), kQTiles), 256, 0, s>>>(p);
    count_launches(1);
    st = check_launch();
  }
  trace_launch_end(WAN_KIND_ATTN, s);
  return st;
}


}  // namespace

int launch_attn_tc(AttnOperand q, AttnOperand k, AttnOperand v, void* o, int64_t o_row_stride, int o_col0, int B,
                   int H, int Lq, int Lk, cudaStream_t s, const SeqScatter* sc, void* scratch, size_t scratch_bytes) {
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
  p.sc = sc ? *sc : SeqScatter{};
  if (sc && (sc->ranks < 1 || sc->ranks > kMaxSeqRanks || sc->rows_local < 1 ||
             static_cast<int64_t>(sc->rows_local) * sc->ranks < Lq))
    return WAN_ERR_SHAPE;
  p.q_scale = nullptr;
  p.kv_scale = nullptr;
  return launch_units<false>(mq, mk, mv, p, B, H, Lq, Lk, s, sc != nullptr, scratch, scratch_bytes);
}

int launch_attn_tc_fp8(const void* q_codes, const float* q_scale, const void* k_codes, const void* vt_codes,
                       int64_t vt_row_stride, const float* kv_scale, void* o, int64_t o_row_stride, int o_col0, int B,
                       int H, int Lq, int Lk, cudaStream_t s, void* scratch, size_t scratch_bytes) {
  if (B == 0 || Lq == 0) return WAN_OK;
  if (Lk <= 0) return WAN_ERR_SHAPE;
  if (vt_row_stride % 16 || vt_row_stride < Lk || o_row_stride % 8 || o_col0 % 8) return WAN_ERR_ALIGN;
  const uint64_t D = static_cast<uint64_t>(H) * kHd;
  // Codes: q [B, Lq, D] and k [B, Lk, D] row-major; v^T [B, D, vt_row_stride] (keys along x).
  CUtensorMap mq, mk, mv;
  const uint64_t dq[3] = {D, static_cast<uint64_t>(Lq), static_cast<uint64_t>(B)};
  const uint64_t sq[2] = {D, D * static_cast<uint64_t>(Lq)};
  const uint64_t dk[3] = {D, static_cast<uint64_t>(Lk), static_cast<uint64_t>(B)};
  const uint64_t sk[2] = {D, D * static_cast<uint64_t>(Lk)};
  const uint64_t dv[3] = {static_cast<uint64_t>(Lk), D, static_cast<uint64_t>(B)};
  const uint64_t sv[2] = {static_cast<uint64_t>(vt_row_stride), static_cast<uint64_t>(vt_row_stride) * D};
  const uint32_t box[3] = {128, kTile, 1};
  if (!make_tmap_u8(&mq, q_codes, 3, dq, sq, box) || !make_tmap_u8(&mk, k_codes, 3, dk, sk, box) ||
      !make_tmap_u8(&mv, vt_codes, 3, dv, sv, box))
    return WAN_ERR_CUDA;
  AttnParams p;
  p.Lq = Lq;
  p.Lk = Lk;
  p.H = H;
  p.q_col0 = 0;
  p.k_col0 = 0;
  p.v_col0 = 0;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(kHd)));
  p.o = static_cast<__nv_bfloat16*>(o);
  p.o_row_stride = o_row_stride;
  p.o_batch_stride = o_row_stride * Lq;
  p.o_col0 = o_col0;
  p.sc = SeqScatter{};
  p.q_scale = q_scale;
  p.kv_scale = kv_scale;
  return launch_units<true>(mq, mk, mv, p, B, H, Lq, Lk, s, false, scratch, scratch_bytes);
}

}  // namespace wan
