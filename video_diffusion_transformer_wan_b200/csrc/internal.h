// Host-side declarations shared by the library's translation units: kernel launchers,
// tensor-map creation, the device error flag and the launch trace.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <mutex>

#include "wan.h"

namespace wan {

// ---------------------------------------------------------------- launch bookkeeping
// Every kernel launch goes through trace_launch_begin/end: they count the launch and,
// when tracing is on, bracket it with CUDA events on the launch stream.
// `work`: algorithmic FLOPs (GEMM, attention) or bytes moved (other kernels).
// Every kernel launch is counted (wan_launch_count): trace_launch_begin counts one;
// launchers that issue more kernels inside one traced bracket, or none, add the rest.
void count_launches(int n);
void trace_launch_begin(int kind, cudaStream_t s, double work = 0.0);
void trace_launch_end(int kind, cudaStream_t s);
int* device_error_flag();   // device address of the error flag of the current device

// Identity (cuCtxGetId) of the calling thread's current CUDA context; false if none.
bool current_context_id(unsigned long long* id);
// Device addresses of one __device__ symbol, one per device, each tagged with the
// context it was looked up in. get() returns the cached address while the device's
// current context is the one it came from, and looks it up again (cudaGetSymbolAddress,
// with the device current) after that context has been replaced, e.g. by a device
// reset that reloads the module at another address.
class SymbolCache {
 public:
  int get(const void* symbol, void** out);

 private:
  static constexpr int kMaxDevices = 64;
  struct Entry {
    void* addr = nullptr;
    unsigned long long ctx = 0;
  };
  Entry entry_[kMaxDevices];
  std::mutex mu_;
};
// One-thread kernel whose bounded wait runs out (about 1 s) and sets the error flag.
int launch_wait_timeout_probe(cudaStream_t s);

// ---------------------------------------------------------------- argument checks
// The checks every entry point applies before any launch (defined in abi.cu).
bool aligned16(const void* p);
int check_ptr(const void* p);       // non-null and 16-byte aligned
int check_opt_ptr(const void* p);   // null, or 16-byte aligned
// Config consistency: dtype, dim == heads * head_dim, multiples of 64, even channel
// counts, freq_dim, eps > 0. `attention`: the call runs attention, which fixes head_dim
// (128 on the bf16 tensor-core path, <= 128 on the fp32 path).
int check_cfg(const wan_dit_config* c, bool attention = false);

// Returns WAN_ERR_CUDA if the last launch failed.
inline int check_launch() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? WAN_OK : WAN_ERR_CUDA;
}

// ---------------------------------------------------------------- tensor maps
// 2D/3D bf16 tile maps with 128-byte swizzle. dims/strides innermost first; strides
// in bytes for dims >= 1. Returns false if the driver rejects the map.
bool make_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                    const uint64_t* strides_bytes, const uint32_t* box);
// The same for 8-bit elements (E4M3 codes).
bool make_tmap_u8(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                  const uint64_t* strides_bytes, const uint32_t* box);
bool make_tmap_f32(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                  const uint64_t* strides_bytes, const uint32_t* box);

// ---------------------------------------------------------------- kernels
// LayerNorm (+ modulation). rows = B*L; e/mod_bias may be NULL (chunk < 0: plain LN).
int launch_layernorm(const float* x, int64_t rows, int D, int L, const float* e, const float* mod_bias,
                     int chunk, void* out, int dtype, float eps, cudaStream_t s);
// The same LN (+ modulation) writing E4M3 codes [rows, D] and one fp32 scale per row
// (amax / 448, 1 for an all-zero row). D in {512, 1536, 5120}; WAN_ERR_UNSUPPORTED else.
int launch_layernorm_e4m3(const float* x, int64_t rows, int D, int L, const float* e, const float* mod_bias,
                          int chunk, void* out, float* row_scale, float eps, cudaStream_t s);

constexpr int kMaxSeqRanks = 8;  // sequence-parallel group size limit

struct GemmEpi {
  int kind;                 // wan_epilogue
  const float* gate;        // RESIDUAL: gate[(m / rows_per_batch) * gate_bstride + n]
  const float* gate_bias;   // RESIDUAL: + gate_bias[n]
  int64_t gate_bstride;
  int rows_per_batch;
  int64_t ldo;              // output row stride (elements)
  // head scatter (kind == kEpiHeadScatter): out[b, c, f, 2i+ph, 2j+pw]
  int sc_F, sc_H, sc_W, sc_C;
  // sequence-parallel scatter (kind == kEpiSeqScatter, a bf16 store): local row
  // m = b*sp_rows_local + i goes to row b*sp_rows_total + sp_row_off + i of rank s's
  // buffer sp_dst[s]; column n = part*sp_part_cols + s*sp_rank_cols + c goes to column
  // part*sp_rank_cols + c there (row stride ldo = parts * sp_rank_cols).
  void* sp_dst[kMaxSeqRanks];
  int sp_rows_local, sp_rows_total, sp_row_off, sp_part_cols, sp_rank_cols;
};
enum : int { kEpiHeadScatter = 100, kEpiSeqScatter = 101 };

// bf16 tcgen05 GEMM: out = epi(A[M,K] W[N,K]^T + bias). A's rows have stride lda
// elements; W has K columns (row stride K). If w_k_period > 0, W has w_k_period
// columns and the k-th reduction index reads W column (k mod w_k_period).
int launch_gemm_tc(const void* A, int64_t lda, const void* W, const void* bias, void* out, int M, int N, int K,
                   int w_k_period, const GemmEpi& epi, cudaStream_t s);
// E4M3 codes of x [M, K] (act dtype, row stride x_stride elements; with sum_halves the
// row is x[:, :K] + x[:, K:2K]) with one scale per row. K, x_stride multiples of 8.
int launch_quantize_rows(const void* x, int64_t x_stride, int M, int K, bool sum_halves, void* q, float* scale,
                         int dtype, cudaStream_t s);
// E4M3 codes of a whole tensor (n elements, multiple of 8) with one scale; scale[0] is
// used as the amax accumulator and holds the scale when the work completes.
int launch_quantize_tensor(const void* x, int64_t n, void* q, float* scale, int dtype, cudaStream_t s);
// E4M3 tcgen05 GEMM (kind::f8f6f4): out = epi(a_scale[m] * w_scale[0] * (A[M,K] W[N,K]^T)
// + bias) with A and W E4M3 codes (row stride lda and K bytes), a_scale [M] and w_scale
// [1] fp32 in device memory. K and lda multiples of 16.
int launch_gemm_e4m3(const void* A, int64_t lda, const float* a_scale, const void* W, const float* w_scale,
                     const void* bias, void* out, int M, int N, int K, const GemmEpi& epi, cudaStream_t s);
// fp32 SIMT GEMM with the same semantics (fp32 activations and weights).
int launch_gemm_simt(const float* A, int64_t lda, const float* W, const float* bias, void* out, int M, int N,
                     int K, int w_k_period, const GemmEpi& epi, cudaStream_t s);

struct AttnOperand {
  const void* ptr;
  int64_t row_stride;  // elements
  int col0;            // column of head 0
};
// Sequence-parallel output scatter: query row l of sample b goes to rank
// r = l / rows_local, row b*rows_local + (l - r*rows_local) of dst[r].
struct SeqScatter {
  int ranks;
  int rows_local;
  void* dst[kMaxSeqRanks];
};
// bf16 tcgen05 flash attention, head_dim 128. With sc, o is ignored and each output row
// is written to its owner's buffer (row stride o_row_stride, columns from o_col0).
// scratch (16-byte aligned, device) lets the last partial wave of work units be split
// over the key tiles; without it (or when too small) every unit runs whole.
int launch_attn_tc(AttnOperand q, AttnOperand k, AttnOperand v, void* o, int64_t o_row_stride, int o_col0,
                   int B, int H, int Lq, int Lk, cudaStream_t s, const SeqScatter* sc = nullptr,
                   void* scratch = nullptr, size_t scratch_bytes = 0);
// 8-bit attention operands from bf16 q, k, v (head_dim 128): q codes [B, Lq, H*128] with
// a scale per (sample, row, head) [B, Lq, H]; k codes [B, Lk, H*128]; v^T codes
// [B, H*128, vt_stride] (vt_stride a multiple of 64, >= Lk; keys past Lk are code 0);
// kv_scale [B, H, 2] = (k scale, v scale). Five kernels.
int launch_attn_fp8_quantize(const void* q, int64_t q_row_stride, int q_col0, const void* k, int64_t k_row_stride,
                             int k_col0, const void* v, int64_t v_row_stride, int v_col0, int B, int H, int Lq, int Lk,
                             void* q_codes, float* q_scale, void* k_codes, void* vt_codes, int64_t vt_stride,
                             float* kv_scale, cudaStream_t s);
// Tensor-core attention over those operands (E4M3 products, E4M3 P); bf16 output.
int launch_attn_tc_fp8(const void* q_codes, const float* q_scale, const void* k_codes, const void* vt_codes,
                       int64_t vt_row_stride, const float* kv_scale, void* o, int64_t o_row_stride, int o_col0, int B,
                       int H, int Lq, int Lk, cudaStream_t s, void* scratch = nullptr, size_t scratch_bytes = 0);
// fp32 SIMT attention, head_dim <= 128, Lk <= 8192.
int launch_attn_simt(AttnOperand q, AttnOperand k, AttnOperand v, void* o, int64_t o_row_stride, int o_col0,
                     int B, int H, int Lq, int Lk, int d, cudaStream_t s);

// Small kernels.
int launch_patch_gather(const void* latent, int B, int C, int F, int H, int W, void* patches, int dtype,
                        cudaStream_t s);
int launch_time_mlp(const float* t, int B, int D, int freq_dim, const void* w1, const void* b1, const void* w2,
                    const void* b2, float* e_out, int dtype, cudaStream_t s, float* hid_scratch = nullptr);
int launch_i2v_input(const void* noise, const void* cond, const uint8_t* keep, int B, int F, int H, int W,
                     void* out, int dtype, cudaStream_t s);
int launch_flow_input(const void* x1, const void* x0, const float* u, int B, int64_t n, void* xt, float* t_out,
                      int dtype, cudaStream_t s);
int launch_sampler_init(const void* input, int B, int64_t n, int64_t in_stride, float* x, void* in2, float* t,
                        int dtype, cudaStream_t s);
int launch_euler_cfg(const float* v, int B, int64_t n, int64_t in_stride, float dt, float g, float* x, void* in2,
                     float* t, float t_next, int dtype, cudaStream_t s, float* delta = nullptr, bool skip = false);
int launch_flow_loss(const float* v, const void* x1, const void* x0, int B, int64_t n, float* loss, int dtype,
                     cudaStream_t s);

inline size_t dtype_size(int dtype) { return dtype == WAN_BF16 ? 2 : 4; }

}  // namespace wan
