// The C ABI (include/wan.h): argument validation, workspace layouts, and the order of
// kernel launches for the Wan 2.1 DiT ("Wan: Open and Advanced Large-Scale Video
// Generative Models"): the block and the stack (section "Diffusion Transformer"), I2V
// and flow matching (sections "I2V 架构扩展", "训练方法"), and the inference paths of
// section "Infra": the guided sampling loop with its diffusion cache, FP8 linear layers,
// and Ulysses sequence parallelism. The host only enqueues work on the caller's stream;
// nothing here allocates device memory. The file runs: device error flag, launch
// trace, tensor maps, validation and workspace layouts, the branch / block / stack
// implementations, then the exported calls.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "internal.h"

namespace wan {

// ------------------------------------------------------------------ module symbols
bool current_context_id(unsigned long long* id) {
  using GetCurrentFn = CUresult (*)(CUcontext*);
  using GetIdFn = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrentFn get_current = nullptr;
  static GetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

int SymbolCache::get(const void* symbol, void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return WAN_ERR_CUDA;
  std::lock_guard<std::mutex> lk(mu_);
  unsigned long long ctx = 0;
  const bool have_ctx = current_context_id(&ctx);
  Entry& en = entry_[dev];
  if (!have_ctx || !en.addr || en.ctx != ctx) {
    void* p = nullptr;
    // Looks the symbol up in this device's current context (creating the runtime's
    // primary context if none exists yet), then records which context that was.
    if (cudaGetSymbolAddress(&p, symbol) != cudaSuccess || !p) return WAN_ERR_CUDA;
    if (!current_context_id(&ctx)) return WAN_ERR_CUDA;
    en.addr = p;
    en.ctx = ctx;
  }
  *out = en.addr;
  return WAN_OK;
}

// ------------------------------------------------------------------ device error flag
__device__ int g_wan_error_flag;

int* device_error_flag() {
  static SymbolCache cache;
  void* p = nullptr;
  return cache.get(&g_wan_error_flag, &p) == WAN_OK ? static_cast<int*>(p) : nullptr;
}

// ------------------------------------------------------------------ trace
namespace {
constexpr int kTracePairs = 16384;
struct Trace {
  std::mutex mu;
  bool on = false;
  std::vector<cudaEvent_t> start, stop;
  std::vector<int> kind;
  std::vector<double> work;
  int used = 0;
};
Trace& trace() {
  static Trace t;
  return t;
}
std::atomic<int64_t> g_launches{0};
thread_local int tl_slot = -1;
}  // namespace

void count_launches(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

void trace_launch_begin(int kind, cudaStream_t s, double work) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  Trace& t = trace();
  tl_slot = -1;
  std::lock_guard<std::mutex> lk(t.mu);
  if (!t.on || t.used >= static_cast<int>(t.start.size())) return;
  tl_slot = t.used++;
  t.kind[tl_slot] = kind;
  t.work[tl_slot] = work;
  cudaEventRecord(t.start[tl_slot], s);
}

void trace_launch_end(int kind, cudaStream_t s) {
  (void)kind;
  if (tl_slot < 0) return;
  Trace& t = trace();
  std::lock_guard<std::mutex> lk(t.mu);
  cudaEventRecord(t.stop[tl_slot], s);
  tl_slot = -1;
}

// ------------------------------------------------------------------ tensor maps
namespace {
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}
}  // namespace

static bool make_tmap(CUtensorMap* map, CUtensorMapDataType type, const void* base, int rank, const uint64_t* dims,
                      const uint64_t* strides_bytes, const uint32_t* box);

bool make_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
                    const uint32_t* box) {
  return make_tmap(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, rank, dims, strides_bytes, box);
}

bool make_tmap_u8(CUtensorMap* map, const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
                  const uint32_t* box) {
  return make_tmap(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, rank, dims, strides_bytes, box);
}

bool make_tmap_f32(CUtensorMap* map, const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
                   const uint32_t* box) {
  return make_tmap(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, base, rank, dims, strides_bytes, box);
}

static bool make_tmap(CUtensorMap* map, CUtensorMapDataType type, const void* base, int rank, const uint64_t* dims,
                      const uint64_t* strides_bytes, const uint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t d[5], st[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
    if (i + 1 < rank) st[i] = strides_bytes[i];
  }
  return fn(map, type, static_cast<cuuint32_t>(rank), const_cast<void*>(base), d, st, bx,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ validation helpers
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define WAN_REQUIRE(cond, code) \
  do {                          \
    if (!(cond)) return (code); \
  } while (0)
#define WAN_TRY(expr)               \
  do {                              \
    int _st = (expr);               \
    if (_st != WAN_OK) return _st;  \
  } while (0)

int check_ptr(const void* p) {
  if (!p) return WAN_ERR_NULL;
  if (!aligned16(p)) return WAN_ERR_ALIGN;
  return WAN_OK;
}
int check_opt_ptr(const void* p) { return p ? check_ptr(p) : WAN_OK; }

namespace {

// Non-null and 4-byte aligned (fp32 scalars and scale vectors).
int check_ptr_any(const void* p) {
  if (!p) return WAN_ERR_NULL;
  return (reinterpret_cast<uintptr_t>(p) & 3u) == 0 ? WAN_OK : WAN_ERR_ALIGN;
}

}  // namespace

int check_cfg(const wan_dit_config* c, bool attention) {
  WAN_REQUIRE(c, WAN_ERR_NULL);
  WAN_REQUIRE(c->dtype == WAN_F32 || c->dtype == WAN_BF16, WAN_ERR_DTYPE);
  WAN_REQUIRE(c->heads > 0 && c->head_dim > 0 && c->dim == c->heads * c->head_dim, WAN_ERR_SHAPE);
  WAN_REQUIRE(c->dim % 64 == 0 && c->ffn_dim > 0 && c->ffn_dim % 64 == 0, WAN_ERR_SHAPE);
  WAN_REQUIRE(c->in_ch > 0 && c->in_ch % 2 == 0 && c->out_ch > 0 && c->out_ch % 2 == 0, WAN_ERR_SHAPE);
  WAN_REQUIRE(c->freq_dim > 0 && c->freq_dim % 8 == 0 && c->freq_dim <= 4096, WAN_ERR_SHAPE);
  WAN_REQUIRE(c->eps > 0.f, WAN_ERR_SHAPE);
  if (!attention) return WAN_OK;
  if (c->dtype == WAN_BF16) {
    WAN_REQUIRE(c->head_dim == 128, WAN_ERR_UNSUPPORTED);
  } else {
    WAN_REQUIRE(c->head_dim <= 128 && c->head_dim % 4 == 0, WAN_ERR_SHAPE);
  }
  return WAN_OK;
}

namespace {

int check_block_w(const wan_dit_config* c, const wan_block_weights* w, bool need_img) {
  WAN_REQUIRE(w, WAN_ERR_NULL);
  WAN_TRY(check_opt_ptr(w->mod_bias));
  const void* req[] = {w->w_qkv, w->w_o, w->w_cq, w->w_ckv, w->w_co, w->w_1, w->w_2};
  for (const void* p : req) WAN_TRY(check_ptr(p));
  const void* opt[] = {w->b_qkv, w->b_o, w->b_cq, w->b_ckv, w->b_co, w->b_1, w->b_2, w->b_ckv_img};
  for (const void* p : opt) WAN_TRY(check_opt_ptr(p));
  if (need_img) WAN_TRY(check_ptr(w->w_ckv_img));
  (void)c;
  return WAN_OK;
}

constexpr size_t kAlign = 256;
size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

struct Layout {
  size_t h;        // [B, L, D] act
  size_t big;      // region R, see below
  size_t x;        // [B, L, D] fp32 (stack)
  size_t e;        // [B, 6, D] fp32 (stack)
  size_t split;    // partial outputs of key-split attention units (see attention())
  size_t split_bytes;
  size_t total;
  size_t big_elems;
};

// Partial outputs for the attention units of a last, less-than-half-full wave that are
// split over their key tiles: per split unit 2 halves x 2 query tiles x 128 rows x
// (128 fp32 + max and sum). At most 74 units (half of 148 SMs) are ever split.
constexpr size_t kSplitUnitBytes = 2 * 2 * 128 * (128 * 4 + 8);
size_t split_bytes(const wan_dit_config* c, int B, int L) {
  const int64_t units = static_cast<int64_t>(B) * c->heads * ((L + 255) / 256);
  return static_cast<size_t>(units < 74 ? units : 74) * kSplitUnitBytes;
}

// Region R (act elements), reused by the three branches:
//   self-attention: qkv [B*L, 3D] at 0, attention output [B*L, D] at 3*B*L*D
//   cross-attention: q [B*L, D] at 0, attention output [B*L, D or 2D] at 3*B*L*D,
//                    text K|V [B*Lc, 2D] at 5*B*L*D, image K|V [B*Li, 2D] after it
//   FFN: hidden [B*L, F] at 0; patchify gather / image MLP scratch also start at 0.
Layout layout(const wan_dit_config* c, int B, int L, int Lc, int Li) {
  const size_t es = dtype_size(c->dtype);
  const size_t D = c->dim, F = c->ffn_dim;
  const size_t BL = static_cast<size_t>(B) * L;
  size_t big = 5 * BL * D + 2 * static_cast<size_t>(B) * (Lc + Li) * D;
  big = big > BL * F ? big : BL * F;
  const size_t patch = BL * c->in_ch * 4;
  big = big > patch ? big : patch;
  const size_t img = 2 * static_cast<size_t>(B) * Li * D;
  big = big > img ? big : img;
  Layout l;
  l.h = 0;
  l.big = align_up(BL * D * es);
  l.big_elems = big;
  l.x = l.big + align_up(big * es);
  l.e = l.x + align_up(BL * D * 4);
  l.split = l.e + align_up(static_cast<size_t>(B) * 6 * D * 4);
  l.split_bytes = c->dtype == WAN_BF16 ? split_bytes(c, B, L) : 0;
  l.total = l.split + align_up(l.split_bytes);
  return l;
}

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }
inline uint8_t* at(void* base, size_t off) { return static_cast<uint8_t*>(base) + off; }

int gemm(const wan_dit_config* c, const void* A, int64_t lda, const void* W, const void* bias, void* out, int M, int N,
         int K, int w_k_period, const GemmEpi& epi, cudaStream_t s) {
  if (c->dtype == WAN_BF16) return launch_gemm_tc(A, lda, W, bias, out, M, N, K, w_k_period, epi, s);
  return launch_gemm_simt(static_cast<const float*>(A), lda, static_cast<const float*>(W),
                          static_cast<const float*>(bias), out, M, N, K, w_k_period, epi, s);
}

int attention(const wan_dit_config* c, AttnOperand q, AttnOperand k, AttnOperand v, void* o, int64_t ors, int oc,
              int B, int Lq, int Lk, cudaStream_t s, void* scratch = nullptr, size_t scratch_bytes = 0) {
  if (c->dtype == WAN_BF16)
    return launch_attn_tc(q, k, v, o, ors, oc, B, c->heads, Lq, Lk, s, nullptr, scratch, scratch_bytes);
  return launch_attn_simt(q, k, v, o, ors, oc, B, c->heads, Lq, Lk, c->head_dim, s);
}

GemmEpi epi_store(int64_t ldo, int kind = WAN_EPI_STORE) {
  GemmEpi e{};
  e.kind = kind;
  e.ldo = ldo;
  e.rows_per_batch = 1;
  return e;
}
GemmEpi epi_residual(int64_t ldo, const float* gate, const float* gate_bias, int64_t bstride, int L) {
  GemmEpi e{};
  e.kind = WAN_EPI_RESIDUAL;
  e.ldo = ldo;
  e.gate = gate;
  e.gate_bias = gate_bias;
  e.gate_bstride = bstride;
  e.rows_per_batch = L;
  return e;
}

// attn_kept: where the attention output goes (and stays, e.g. across sampling steps), or
// NULL for the workspace; with attn_reuse the kept output is used as it is and neither
// the QKV projection nor the attention runs.
int self_attn_impl(const wan_dit_config* c, const void* h, const wan_block_weights* w, const float* e, float* x, int B,
                   int L, void* ws, const Layout& ly, cudaStream_t s, void* attn_kept = nullptr,
                   bool attn_reuse = false) {
  const int D = c->dim;
  const size_t es = dtype_size(c->dtype);
  const int M = B * L;
  uint8_t* R = at(ws, ly.big);
  void* qkv = R;
  void* o = attn_kept ? attn_kept : R + static_cast<size_t>(3) * M * D * es;
  if (!(attn_kept && attn_reuse)) {
    WAN_TRY(gemm(c, h, D, w->w_qkv, w->b_qkv, qkv, M, 3 * D, D, 0, epi_store(3 * D), s));
    WAN_TRY(attention(c, {qkv, 3 * D, 0}, {qkv, 3 * D, D}, {qkv, 3 * D, 2 * D}, o, D, 0, B, L, L, s,
                      at(ws, ly.split), ly.split_bytes));
  }
  const float* gb = w->mod_bias ? w->mod_bias + 2 * D : nullptr;
  return gemm(c, o, D, w->w_o, w->b_o, x, M, D, D, 0, epi_residual(D, e + 2 * D, gb, 6 * D, L), s);
}

// kvt_cached / kvi_cached: text / image K|V already projected ([B*Lc, 2D], [B*Li, 2D]
// act), e.g. kept across sampling steps; the projections are skipped when given.
int cross_attn_impl(const wan_dit_config* c, const void* h, const void* ctx, int Lc, const void* img, int Li,
                    const wan_block_weights* w, float* x, int B, int L, void* ws, const Layout& ly, cudaStream_t s,
                    const void* kvt_cached = nullptr, const void* kvi_cached = nullptr) {
  if (B == 0 || L == 0) return WAN_OK;  // no query rows: nothing to add to x
  const int D = c->dim;
  const size_t es = dtype_size(c->dtype);
  const int M = B * L;
  uint8_t* R = at(ws, ly.big);
  void* q = R;
  void* ocat = R + static_cast<size_t>(3) * M * D * es;
  void* kvt = R + static_cast<size_t>(5) * M * D * es;
  void* kvi = static_cast<uint8_t*>(kvt) + static_cast<size_t>(2) * B * Lc * D * es;
  const bool with_img = img && Li > 0;
  const int ow = with_img ? 2 * D : D;
  WAN_TRY(gemm(c, h, D, w->w_cq, w->b_cq, q, M, D, D, 0, epi_store(D), s));
  if (kvt_cached)
    kvt = const_cast<void*>(kvt_cached);
  else
    WAN_TRY(gemm(c, ctx, D, w->w_ckv, w->b_ckv, kvt, B * Lc, 2 * D, D, 0, epi_store(2 * D), s));
  void* scr = at(ws, ly.split);
  const size_t scr_bytes = ly.split_bytes;
  WAN_TRY(attention(c, {q, D, 0}, {kvt, 2 * D, 0}, {kvt, 2 * D, D}, ocat, ow, 0, B, L, Lc, s, scr, scr_bytes));
  if (with_img) {
    if (kvi_cached)
      kvi = const_cast<void*>(kvi_cached);
    else
      WAN_TRY(gemm(c, img, D, w->w_ckv_img, w->b_ckv_img, kvi, B * Li, 2 * D, D, 0, epi_store(2 * D), s));
    WAN_TRY(attention(c, {q, D, 0}, {kvi, 2 * D, 0}, {kvi, 2 * D, D}, ocat, ow, D, B, L, Li, s, scr, scr_bytes));
    // (o_text + o_image) Wco^T as one reduction over [o_text | o_image] with Wco reused.
    return gemm(c, ocat, ow, w->w_co, w->b_co, x, M, D, 2 * D, D, epi_residual(D, nullptr, nullptr, 0, L), s);
  }
  return gemm(c, ocat, D, w->w_co, w->b_co, x, M, D, D, 0, epi_residual(D, nullptr, nullptr, 0, L), s);
}

int ffn_impl(const wan_dit_config* c, const void* h, const wan_block_weights* w, const float* e, float* x, int B, int L,
             void* ws, const Layout& ly, cudaStream_t s) {
  const int D = c->dim, F = c->ffn_dim;
  const int M = B * L;
  void* hid = at(ws, ly.big);
  WAN_TRY(gemm(c, h, D, w->w_1, w->b_1, hid, M, F, D, 0, epi_store(F, WAN_EPI_GELU), s));
  const float* gb = w->mod_bias ? w->mod_bias + 5 * D : nullptr;
  return gemm(c, hid, F, w->w_2, w->b_2, x, M, D, F, 0, epi_residual(D, e + 5 * D, gb, 6 * D, L), s);
}

int block_impl(const wan_dit_config* c, float* x, const float* e, const void* ctx, int Lc, const void* img, int Li,
               const wan_block_weights* w, int B, int L, void* ws, const Layout& ly, cudaStream_t s,
               const void* kvt_cached = nullptr, const void* kvi_cached = nullptr, void* attn_kept = nullptr,
               bool attn_reuse = false) {
  if (B == 0 || L == 0) return WAN_OK;
  void* h = at(ws, ly.h);
  const int64_t rows = static_cast<int64_t>(B) * L;
  WAN_TRY(launch_layernorm(x, rows, c->dim, L, e, w->mod_bias, 0, h, c->dtype, c->eps, s));
  WAN_TRY(self_attn_impl(c, h, w, e, x, B, L, ws, ly, s, attn_kept, attn_reuse));
  WAN_TRY(launch_layernorm(x, rows, c->dim, L, nullptr, nullptr, -1, h, c->dtype, c->eps, s));
  WAN_TRY(cross_attn_impl(c, h, ctx, Lc, img, Li, w, x, B, L, ws, ly, s, kvt_cached, kvi_cached));
  WAN_TRY(launch_layernorm(x, rows, c->dim, L, e, w->mod_bias, 1, h, c->dtype, c->eps, s));
  return ffn_impl(c, h, w, e, x, B, L, ws, ly, s);
}

// Plain LN of the residual stream, then Linear(D, out_ch*4) whose epilogue scatters each
// token's (c, ph, pw) outputs into the unpatchified latent.
int head_impl(const wan_dit_config* c, const float* x, int B, int F, int H, int W, const void* w_head,
              const void* b_head, float* v_out, void* h, cudaStream_t s) {
  const int L = F * (H / 2) * (W / 2);
  WAN_TRY(launch_layernorm(x, static_cast<int64_t>(B) * L, c->dim, L, nullptr, nullptr, -1, h, c->dtype, c->eps, s));
  GemmEpi ep{};
  ep.kind = kEpiHeadScatter;
  ep.rows_per_batch = L;
  ep.sc_C = c->out_ch;
  ep.sc_F = F;
  ep.sc_H = H;
  ep.sc_W = W;
  return gemm(c, h, c->dim, w_head, b_head, v_out, B * L, c->out_ch * 4, c->dim, 0, ep, s);
}

// FP8 (E4M3) block
// FP8 block workspace: the bf16 block's layout (its h region unused), then E4M3 codes
// of the block inputs ([B*L, max(D, F)], reused by each linear layer in turn), codes of
// the text / image context ([B*max(Lc, Li), D]) and the per-row scales of both.
// 8-bit attention workspace: q codes, q scales, k codes, v^T codes, k/v scales, and the
// key-split scratch of a partial last wave.
struct AttnF8Layout {
  size_t qc, qs, kc, vt, kvs, split, split_bytes, total;
  int64_t vt_stride;
};
AttnF8Layout attn_f8_layout(const wan_dit_config* c, int B, int Lq, int Lk) {
  const size_t D = c->dim, H = c->heads;
  AttnF8Layout l;
  l.vt_stride = (static_cast<int64_t>(Lk) + 63) / 64 * 64;
  l.qc = 0;
  l.qs = l.qc + align_up(static_cast<size_t>(B) * Lq * D);
  l.kc = l.qs + align_up(static_cast<size_t>(B) * Lq * H * 4);
  l.vt = l.kc + align_up(static_cast<size_t>(B) * Lk * D);
  l.kvs = l.vt + align_up(static_cast<size_t>(B) * D * l.vt_stride);
  l.split = l.kvs + align_up(static_cast<size_t>(B) * H * 2 * 4);
  l.split_bytes = split_bytes(c, B, Lq);
  l.total = l.split + align_up(l.split_bytes);
  return l;
}

struct Fp8Layout {
  Layout base;
  size_t codes, ctx_codes, scales, ctx_scales, attn, total;
  AttnF8Layout attn_parts;  // offsets relative to `attn` (its own key-split scratch unused)
};
Fp8Layout fp8_layout(const wan_dit_config* c, int B, int L, int Lc, int Li) {
  Fp8Layout l;
  l.base = layout(c, B, L, Lc, Li);
  const size_t BL = static_cast<size_t>(B) * L;
  const size_t Lx = static_cast<size_t>(B) * (Lc > Li ? Lc : Li);
  const size_t wmax = c->ffn_dim > c->dim ? c->ffn_dim : c->dim;
  l.codes = l.base.total;
  l.ctx_codes = l.codes + align_up(BL * wmax);
  l.scales = l.ctx_codes + align_up(Lx * c->dim);
  l.ctx_scales = l.scales + align_up(BL * 4);
  // operands of 8-bit self-attention (used when the scales ask for it)
  l.attn = l.ctx_scales + align_up(Lx * 4);
  l.attn_parts = attn_f8_layout(c, B, L, L);
  l.total = l.attn + align_up(l.attn_parts.split);
  return l;
}

int check_scales(const wan_fp8_scales* sc, bool with_img) {
  WAN_REQUIRE(sc, WAN_ERR_NULL);
  WAN_TRY(check_ptr_any(sc->qkv));
  WAN_TRY(check_ptr_any(sc->o));
  WAN_TRY(check_ptr_any(sc->cq));
  WAN_TRY(check_ptr_any(sc->ckv));
  WAN_TRY(check_ptr_any(sc->co));
  WAN_TRY(check_ptr_any(sc->ffn1));
  WAN_TRY(check_ptr_any(sc->ffn2));
  if (with_img) WAN_TRY(check_ptr_any(sc->ckv_img));
  return WAN_OK;
}

int e4m3_gemm(const void* A, const float* as, const void* W, const float* wsc, const void* bias, void* out, int M,
              int N, int K, const GemmEpi& ep, cudaStream_t s) {
  return launch_gemm_e4m3(A, K, as, W, wsc, bias, out, M, N, K, ep, s);
}
int block_fp8_impl(const wan_dit_config* cfg, float* x, const float* e, const void* ctx, int Lc, const void* img_ctx,
                   int li, const wan_block_weights* w, const wan_fp8_scales* sc, int B, int L, void* workspace,
                   const Fp8Layout& fl, cudaStream_t s, const void* kvt_cached = nullptr,
                   const void* kvi_cached = nullptr, void* attn_kept = nullptr, bool attn_reuse = false) {
  const bool with_img = img_ctx && li > 0;
  const int D = cfg->dim, Fd = cfg->ffn_dim;
  const int M = B * L;
  const int64_t rows = M;
  uint8_t* R = at(workspace, fl.base.big);
  void* codes = at(workspace, fl.codes);
  void* ctx_codes = at(workspace, fl.ctx_codes);
  float* scales = reinterpret_cast<float*>(at(workspace, fl.scales));
  float* ctx_scales = reinterpret_cast<float*>(at(workspace, fl.ctx_scales));
  const size_t MD = static_cast<size_t>(M) * D * 2;  // bytes of one [M, D] bf16 slab
  // self-attention
  WAN_TRY(launch_layernorm_e4m3(x, rows, D, L, e, w->mod_bias, 0, codes, scales, cfg->eps, s));
  void* qkv = R;
  void* o = attn_kept ? attn_kept : R + 3 * MD;
  void* scr = at(workspace, fl.base.split);
  const size_t scr_bytes = fl.base.split_bytes;
  if (!(attn_kept && attn_reuse)) {
    WAN_TRY(e4m3_gemm(codes, scales, w->w_qkv, sc->qkv, w->b_qkv, qkv, M, 3 * D, D, epi_store(3 * D), s));
    if (sc->attention_fp8) {
      const AttnF8Layout& a = fl.attn_parts;
      uint8_t* A = at(workspace, fl.attn);
      float* qs = reinterpret_cast<float*>(A + a.qs);
      float* kvs = reinterpret_cast<float*>(A + a.kvs);
      WAN_TRY(launch_attn_fp8_quantize(qkv, 3 * D, 0, qkv, 3 * D, D, qkv, 3 * D, 2 * D, B, cfg->heads, L, L, A + a.qc,
                                       qs, A + a.kc, A + a.vt, a.vt_stride, kvs, s));
      WAN_TRY(launch_attn_tc_fp8(A + a.qc, qs, A + a.kc, A + a.vt, a.vt_stride, kvs, o, D, 0, B, cfg->heads, L, L, s,
                                 scr, scr_bytes));
    } else {
      WAN_TRY(launch_attn_tc({qkv, 3 * D, 0}, {qkv, 3 * D, D}, {qkv, 3 * D, 2 * D}, o, D, 0, B, cfg->heads, L, L, s,
                             nullptr, scr, scr_bytes));
    }
  }
  WAN_TRY(launch_quantize_rows(o, D, M, D, false, codes, scales, WAN_BF16, s));
  const float* gb_msa = w->mod_bias ? w->mod_bias + 2 * D : nullptr;
  WAN_TRY(e4m3_gemm(codes, scales, w->w_o, sc->o, w->b_o, x, M, D, D, epi_residual(D, e + 2 * D, gb_msa, 6 * D, L), s));
  // cross-attention
  WAN_TRY(launch_layernorm_e4m3(x, rows, D, L, nullptr, nullptr, -1, codes, scales, cfg->eps, s));
  void* q = R;
  void* ocat = R + 3 * MD;
  void* kvt = R + 5 * MD;
  void* kvi = static_cast<uint8_t*>(kvt) + static_cast<size_t>(B) * Lc * 2 * D * 2;
  WAN_TRY(e4m3_gemm(codes, scales, w->w_cq, sc->cq, w->b_cq, q, M, D, D, epi_store(D), s));
  if (kvt_cached) {
    kvt = const_cast<void*>(kvt_cached);
  } else {
    WAN_TRY(launch_quantize_rows(ctx, D, B * Lc, D, false, ctx_codes, ctx_scales, WAN_BF16, s));
    WAN_TRY(e4m3_gemm(ctx_codes, ctx_scales, w->w_ckv, sc->ckv, w->b_ckv, kvt, B * Lc, 2 * D, D, epi_store(2 * D),
                      s));
  }
  const int ow = with_img ? 2 * D : D;
  WAN_TRY(launch_attn_tc({q, D, 0}, {kvt, 2 * D, 0}, {kvt, 2 * D, D}, ocat, ow, 0, B, cfg->heads, L, Lc, s, nullptr,
                         scr, scr_bytes));
  if (with_img) {
    if (kvi_cached) {
      kvi = const_cast<void*>(kvi_cached);
    } else {
      WAN_TRY(launch_quantize_rows(img_ctx, D, B * li, D, false, ctx_codes, ctx_scales, WAN_BF16, s));
      WAN_TRY(e4m3_gemm(ctx_codes, ctx_scales, w->w_ckv_img, sc->ckv_img, w->b_ckv_img, kvi, B * li, 2 * D, D,
                        epi_store(2 * D), s));
    }
    WAN_TRY(launch_attn_tc({q, D, 0}, {kvi, 2 * D, 0}, {kvi, 2 * D, D}, ocat, ow, D, B, cfg->heads, L, li, s,
                           nullptr, scr, scr_bytes));
  }
  // the text and image outputs are summed while quantised
  WAN_TRY(launch_quantize_rows(ocat, ow, M, D, with_img, codes, scales, WAN_BF16, s));
  WAN_TRY(e4m3_gemm(codes, scales, w->w_co, sc->co, w->b_co, x, M, D, D, epi_residual(D, nullptr, nullptr, 0, L), s));
  // FFN
  WAN_TRY(launch_layernorm_e4m3(x, rows, D, L, e, w->mod_bias, 1, codes, scales, cfg->eps, s));
  void* hid = R;
  WAN_TRY(e4m3_gemm(codes, scales, w->w_1, sc->ffn1, w->b_1, hid, M, Fd, D, epi_store(Fd, WAN_EPI_GELU), s));
  WAN_TRY(launch_quantize_rows(hid, Fd, M, Fd, false, codes, scales, WAN_BF16, s));
  const float* gb_ffn = w->mod_bias ? w->mod_bias + 5 * D : nullptr;
  return e4m3_gemm(codes, scales, w->w_2, sc->ffn2, w->b_2, x, M, D, Fd,
                   epi_residual(D, e + 5 * D, gb_ffn, 6 * D, L), s);
}

// patchify -> timestep MLP -> blocks -> head. kvt/kvi: per-block cached cross-attention
// K|V (arrays of n_blocks pointers) or NULL.
int stack_impl(const wan_dit_config* cfg, int n_blocks, const void* latent, int B, int F, int H, int W,
               const float* t, const wan_stack_weights* sw, const wan_block_weights* blocks, const void* ctx, int Lc,
               const void* img_ctx, int li, float* v_out, void* workspace, const Layout& ly, cudaStream_t s,
               const void* const* kvt, const void* const* kvi, void* const* attn_kept = nullptr,
               bool attn_reuse = false, const wan_fp8_scales* fp8 = nullptr, const Fp8Layout* fl = nullptr) {
  const int L = F * (H / 2) * (W / 2);
  float* x = reinterpret_cast<float*>(at(workspace, ly.x));
  float* e = reinterpret_cast<float*>(at(workspace, ly.e));
  void* patches = at(workspace, ly.big);
  const int K = cfg->in_ch * 4;
  WAN_TRY(launch_patch_gather(latent, B, cfg->in_ch, F, H, W, patches, cfg->dtype, s));
  WAN_TRY(gemm(cfg, patches, K, sw->w_p, sw->b_p, x, B * L, cfg->dim, K, 0, epi_store(cfg->dim, WAN_EPI_F32), s));
  // the hidden units of the time MLP go to region R, free once the patchify GEMM has run
  WAN_TRY(launch_time_mlp(t, B, cfg->dim, cfg->freq_dim, sw->time.w_t1, sw->time.b_t1, sw->time.w_t2, sw->time.b_t2,
                          e, cfg->dtype, s, reinterpret_cast<float*>(patches)));
  for (int i = 0; i < n_blocks; ++i) {
    const void* kt = kvt ? kvt[i] : nullptr;
    const void* ki = kvi ? kvi[i] : nullptr;
    void* kept = attn_kept ? attn_kept[i] : nullptr;
    if (fp8)
      WAN_TRY(block_fp8_impl(cfg, x, e, ctx, Lc, img_ctx, li, &blocks[i], &fp8[i], B, L, workspace, *fl, s, kt, ki,
                             kept, attn_reuse));
    else
      WAN_TRY(block_impl(cfg, x, e, ctx, Lc, img_ctx, li, &blocks[i], B, L, workspace, ly, s, kt, ki, kept,
                         attn_reuse));
  }
  return head_impl(cfg, x, B, F, H, W, sw->w_head, sw->b_head, v_out, at(workspace, ly.h), s);
}

// Sampler workspace: the stack's workspace for 2B samples, the 2B-sample DiT input, the
// 2B velocities (fp32), the 2B timesteps, and per block the cached text and image K|V
// of both contexts.
struct SampleLayout {
  size_t in2, v, t, kvt, kvi, attn, delta, total;
  size_t kvt_block, kvi_block, attn_block;  // bytes per block
};
SampleLayout sample_layout(const wan_dit_config* c, int n_blocks, int B, int F, int H, int W, int Lc, int Li,
                           bool cache, bool fp8) {
  const size_t es = dtype_size(c->dtype);
  const int L = F * (H / 2) * (W / 2);
  const size_t fhw = static_cast<size_t>(F) * H * W;
  SampleLayout l;
  l.in2 = align_up(fp8 ? fp8_layout(c, 2 * B, L, Lc, Li).total : layout(c, 2 * B, L, Lc, Li).total);
  l.v = l.in2 + align_up(2 * static_cast<size_t>(B) * c->in_ch * fhw * es);
  l.t = l.v + align_up(2 * static_cast<size_t>(B) * c->out_ch * fhw * 4);
  l.kvt = l.t + align_up(2 * static_cast<size_t>(B) * 4);
  l.kvt_block = align_up(2 * static_cast<size_t>(B) * Lc * 2 * c->dim * es);
  l.kvi_block = align_up(2 * static_cast<size_t>(B) * Li * 2 * c->dim * es);
  l.kvi = l.kvt + static_cast<size_t>(n_blocks) * l.kvt_block;
  l.attn = l.kvi + static_cast<size_t>(n_blocks) * l.kvi_block;
  l.attn_block = cache ? align_up(2 * static_cast<size_t>(B) * L * c->dim * es) : 0;
  l.delta = l.attn + static_cast<size_t>(n_blocks) * l.attn_block;
  l.total = l.delta + (cache ? align_up(static_cast<size_t>(B) * c->out_ch * fhw * 4) : 0);
  return l;
}

int check_tokens(const wan_dit_config* c, int B, int L, int Lc, int Li) {
  WAN_REQUIRE(B >= 0 && L >= 0 && Lc >= 0 && Li >= 0, WAN_ERR_SHAPE);
  WAN_REQUIRE(static_cast<int64_t>(B) * L < (int64_t(1) << 31), WAN_ERR_SHAPE);
  if (c->dtype == WAN_F32) WAN_REQUIRE(L <= 8192 && Lc <= 8192 && Li <= 8192, WAN_ERR_SHAPE);
  return WAN_OK;
}

int check_ws(const wan_dit_config* c, void* ws, size_t ws_bytes, int B, int L, int Lc, int Li) {
  WAN_TRY(check_ptr(ws));
  WAN_REQUIRE(ws_bytes >= layout(c, B, L, Lc, Li).total, WAN_ERR_WORKSPACE);
  return WAN_OK;
}

}  // namespace
}  // namespace wan

using namespace wan;

extern "C" {

const char* wan_status_string(int status) {
  switch (status) {
    case WAN_OK: return "ok";
    case WAN_ERR_NULL: return "a required pointer is NULL";
    case WAN_ERR_SHAPE: return "sizes inconsistent or outside the supported range";
    case WAN_ERR_DTYPE: return "unknown dtype";
    case WAN_ERR_ALIGN: return "a device pointer or stride is not 16-byte aligned";
    case WAN_ERR_WORKSPACE: return "workspace smaller than wan_workspace_bytes()";
    case WAN_ERR_CUDA: return "a CUDA launch or runtime call failed";
    case WAN_ERR_TIMEOUT: return "a bounded device-side wait ran out";
    case WAN_ERR_UNSUPPORTED: return "request not implemented by this build";
    default: return "unknown status";
  }
}

size_t wan_workspace_bytes(const wan_dit_config* cfg, int B, int L, int Lc, int Li) {
  if (check_cfg(cfg) != WAN_OK || B < 0 || L < 0 || Lc < 0 || Li < 0) return 0;
  return layout(cfg, B, L, Lc, Li).total;
}

int wan_wait_timeout_check(void* stream) { return launch_wait_timeout_probe(as_stream(stream)); }

int wan_device_status(void* stream) {
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return WAN_ERR_CUDA;
  int* flag = device_error_flag();
  if (!flag) return WAN_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, flag, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return WAN_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    cudaMemcpy(flag, &zero, sizeof(int), cudaMemcpyHostToDevice);
    return WAN_ERR_TIMEOUT;
  }
  return WAN_OK;
}

int wan_patchify(const wan_dit_config* cfg, const void* latent, int B, int F, int H, int W, const void* w_p,
                 const void* b_p, float* x_out, void* workspace, size_t ws_bytes, void* stream) {
  WAN_TRY(check_cfg(cfg));
  WAN_TRY(check_ptr(latent));
  WAN_TRY(check_ptr(w_p));
  WAN_TRY(check_opt_ptr(b_p));
  WAN_TRY(check_ptr(x_out));
  WAN_TRY(check_ptr(workspace));
  WAN_REQUIRE(B >= 0 && F >= 0 && H >= 0 && W >= 0 && H % 2 == 0 && W % 2 == 0, WAN_ERR_SHAPE);
  const size_t rows = static_cast<size_t>(B) * F * (H / 2) * (W / 2);
  WAN_REQUIRE(rows < (size_t(1) << 31), WAN_ERR_SHAPE);
  const int K = cfg->in_ch * 4;
  WAN_REQUIRE(ws_bytes >= rows * K * dtype_size(cfg->dtype), WAN_ERR_WORKSPACE);
  cudaStream_t s = as_stream(stream);
  WAN_TRY(launch_patch_gather(latent, B, cfg->in_ch, F, H, W, workspace, cfg->dtype, s));
  return gemm(cfg, workspace, K, w_p, b_p, x_out, static_cast<int>(rows), cfg->dim, K, 0,
              epi_store(cfg->dim, WAN_EPI_F32), s);
}

int wan_time_mlp(const wan_dit_config* cfg, const float* t, int B, const wan_time_weights* w, float* e_out,
                 void* stream) {
  WAN_TRY(check_cfg(cfg));
  WAN_REQUIRE(w, WAN_ERR_NULL);
  WAN_TRY(check_ptr(t));
  WAN_TRY(check_ptr(w->w_t1));
  WAN_TRY(check_ptr(w->w_t2));
  WAN_TRY(check_ptr(w->b_t1));
  WAN_TRY(check_ptr(w->b_t2));
  WAN_TRY(check_ptr(e_out));
  WAN_REQUIRE(B >= 0, WAN_ERR_SHAPE);
  return launch_time_mlp(t, B, cfg->dim, cfg->freq_dim, w->w_t1, w->b_t1, w->w_t2, w->b_t2, e_out, cfg->dtype,
                         as_stream(stream));
}

int wan_adaln_modulate(const wan_dit_config* cfg, const float* x, int B, int L, const float* e, const float* mod_bias,
                       int chunk, void* h_out, void* stream) {
  WAN_TRY(check_cfg(cfg));
  WAN_TRY(check_ptr(x));
  WAN_TRY(check_ptr(h_out));
  WAN_REQUIRE(chunk >= -1 && chunk <= 1 && B >= 0 && L >= 0, WAN_ERR_SHAPE);
  if (chunk >= 0) WAN_TRY(check_ptr(e));
  WAN_TRY(check_opt_ptr(mod_bias));
  return launch_layernorm(x, static_cast<int64_t>(B) * L, cfg->dim, L, e, mod_bias, chunk, h_out, cfg->dtype,
                          cfg->eps, as_stream(stream));
}

int wan_self_attn_fwd(const wan_dit_config* cfg, const void* h, const wan_block_weights* w, const float* e,
                      float* x_inout, int B, int L, void* workspace, size_t ws_bytes, void* stream) {
  WAN_TRY(check_cfg(cfg, true));
  WAN_TRY(check_block_w(cfg, w, false));
  WAN_TRY(check_ptr(h));
  WAN_TRY(check_ptr(e));
  WAN_TRY(check_ptr(x_inout));
  WAN_TRY(check_tokens(cfg, B, L, 0, 0));
  WAN_TRY(check_ws(cfg, workspace, ws_bytes, B, L, 0, 0));
  return self_attn_impl(cfg, h, w, e, x_inout, B, L, workspace, layout(cfg, B, L, 0, 0), as_stream(stream));
}

int wan_cross_attn_fwd(const wan_dit_config* cfg, const void* h, const void* ctx, int Lc, const void* img_ctx, int Li,
                       const wan_block_weights* w, float* x_inout, int B, int L, void* workspace, size_t ws_bytes,
                       void* stream) {
  WAN_TRY(check_cfg(cfg, true));
  const bool with_img = img_ctx && Li > 0;
  WAN_TRY(check_block_w(cfg, w, with_img));
  WAN_TRY(check_ptr(h));
  WAN_TRY(check_ptr(ctx));
  WAN_TRY(check_opt_ptr(img_ctx));
  WAN_TRY(check_ptr(x_inout));
  WAN_REQUIRE(Lc > 0, WAN_ERR_SHAPE);
  WAN_TRY(check_tokens(cfg, B, L, Lc, Li));
  WAN_TRY(check_ws(cfg, workspace, ws_bytes, B, L, Lc, with_img ? Li : 0));
  return cross_attn_impl(cfg, h, ctx, Lc, img_ctx, with_img ? Li : 0, w, x_inout, B, L, workspace,
                         layout(cfg, B, L, Lc, with_img ? Li : 0), as_stream(stream));
}

int wan_ffn_fwd(const wan_dit_config* cfg, const void* h, const wan_block_weights* w, const float* e, float* x_inout,
                int B, int L, void* workspace, size_t ws_bytes, void* stream) {
  WAN_TRY(check_cfg(cfg));
  WAN_TRY(check_block_w(cfg, w, false));
  WAN_TRY(check_ptr(h));
  WAN_TRY(check_ptr(e));
  WAN_TRY(check_ptr(x_inout));
  WAN_TRY(check_tokens(cfg, B, L, 0, 0));
  WAN_TRY(check_ws(cfg, workspace, ws_bytes, B, L, 0, 0));
  return ffn_impl(cfg, h, w, e, x_inout, B, L, workspace, layout(cfg, B, L, 0, 0), as_stream(stream));
}

int wan_dit_block_fwd(const wan_dit_config* cfg, float* x_inout, const float* e, const void* ctx, int Lc,
                      const void* img_ctx, int Li, const wan_block_weights* w, int B, int L, void* workspace,
                      size_t ws_bytes, void* stream) {
  WAN_TRY(check_cfg(cfg, true));
  const bool with_img = img_ctx && Li > 0;
  WAN_TRY(check_block_w(cfg, w, with_img));
  WAN_TRY(check_ptr(x_inout));
  WAN_TRY(check_ptr(e));
  WAN_TRY(check_ptr(ctx));
  WAN_TRY(check_opt_ptr(img_ctx));
  WAN_REQUIRE(Lc > 0, WAN_ERR_SHAPE);
  WAN_TRY(check_tokens(cfg, B, L, Lc, Li));
  const int li = with_img ? Li : 0;
  WAN_TRY(check_ws(cfg, workspace, ws_bytes, B, L, Lc, li));
  return block_impl(cfg, x_inout, e, ctx, Lc, img_ctx, li, w, B, L, workspace, layout(cfg, B, L, Lc, li),
                    as_stream(stream));
}

int wan_dit_stack_fwd(const wan_dit_config* cfg, int n_blocks, const void* latent, int B, int F, int H, int W,
                      const float* t, const wan_stack_weights* sw, const wan_block_weights* blocks, const void* ctx,
                      int Lc, const void* img_ctx, int Li, float* v_out, void* workspace, size_t ws_bytes,
                      void* stream) {
  WAN_TRY(check_cfg(cfg, true));
  WAN_REQUIRE(sw && (blocks || n_blocks == 0), WAN_ERR_NULL);
  WAN_REQUIRE(n_blocks >= 0, WAN_ERR_SHAPE);
  WAN_REQUIRE(B >= 0 && F >= 0 && H % 2 == 0 && W % 2 == 0 && H >= 0 && W >= 0, WAN_ERR_SHAPE);
  const bool with_img = img_ctx && Li > 0;
  for (int i = 0; i < n_blocks; ++i) WAN_TRY(check_block_w(cfg, &blocks[i], with_img));
  WAN_TRY(check_ptr(latent));
  WAN_TRY(check_ptr(t));
  WAN_TRY(check_ptr(ctx));
  WAN_TRY(check_opt_ptr(img_ctx));
  WAN_TRY(check_ptr(v_out));
  WAN_TRY(check_ptr(sw->w_p));
  WAN_TRY(check_opt_ptr(sw->b_p));
  WAN_TRY(check_ptr(sw->w_head));
  WAN_TRY(check_opt_ptr(sw->b_head));
  WAN_TRY(check_ptr(sw->time.w_t1));
  WAN_TRY(check_ptr(sw->time.w_t2));
  WAN_TRY(check_ptr(sw->time.b_t1));
  WAN_TRY(check_ptr(sw->time.b_t2));
  WAN_REQUIRE(Lc > 0, WAN_ERR_SHAPE);
  const int L = F * (H / 2) * (W / 2);
  const int li = with_img ? Li : 0;
  WAN_TRY(check_tokens(cfg, B, L, Lc, li));
  WAN_TRY(check_ws(cfg, workspace, ws_bytes, B, L, Lc, li));
  return stack_impl(cfg, n_blocks, latent, B, F, H, W, t, sw, blocks, ctx, Lc, img_ctx, li, v_out, workspace,
                    layout(cfg, B, L, Lc, li), as_stream(stream), nullptr, nullptr);
}

namespace {
int check_sp(const wan_dit_config* cfg, int P, int r, int B, int L, void* const* ptrs) {
  WAN_TRY(check_cfg(cfg, true));
  if (cfg->dtype != WAN_BF16) return WAN_ERR_UNSUPPORTED;
  WAN_REQUIRE(P >= 1 && P <= kMaxSeqRanks && r >= 0 && r < P, WAN_ERR_SHAPE);
  WAN_REQUIRE(cfg->heads % P == 0 && B >= 0 && L >= 0 && L % P == 0, WAN_ERR_SHAPE);
  WAN_REQUIRE(ptrs, WAN_ERR_NULL);
  for (int s = 0; s < P; ++s) WAN_TRY(check_ptr(ptrs[s]));
  return check_tokens(cfg, B, L, 0, 0);
}
}  // namespace

int wan_sp_qkv_fwd(const wan_dit_config* cfg, int sp_size, int sp_rank, const void* h, int B, int L,
                   const wan_block_weights* w, void* const* qkv_dst, void* stream) {
  WAN_TRY(check_sp(cfg, sp_size, sp_rank, B, L, qkv_dst));
  WAN_REQUIRE(w, WAN_ERR_NULL);
  WAN_TRY(check_ptr(w->w_qkv));
  WAN_TRY(check_opt_ptr(w->b_qkv));
  WAN_TRY(check_ptr(h));
  const int D = cfg->dim, Ll = L / sp_size;
  if (B == 0 || L == 0) return WAN_OK;
  GemmEpi ep = epi_store(3 * D / sp_size);
  ep.kind = kEpiSeqScatter;
  for (int s = 0; s < sp_size; ++s) ep.sp_dst[s] = qkv_dst[s];
  ep.sp_rows_local = Ll;
  ep.sp_rows_total = L;
  ep.sp_row_off = sp_rank * Ll;
  ep.sp_part_cols = D;
  ep.sp_rank_cols = D / sp_size;
  return gemm(cfg, h, D, w->w_qkv, w->b_qkv, nullptr, B * Ll, 3 * D, D, 0, ep, as_stream(stream));
}

int wan_sp_attn_fwd(const wan_dit_config* cfg, int sp_size, int sp_rank, const void* qkv, int B, int L,
                    void* const* o_dst, void* stream) {
  WAN_TRY(check_sp(cfg, sp_size, sp_rank, B, L, o_dst));
  WAN_TRY(check_ptr(qkv));
  const int D = cfg->dim, Dl = D / sp_size;
  if (B == 0 || L == 0) return WAN_OK;
  SeqScatter sc{};
  sc.ranks = sp_size;
  sc.rows_local = L / sp_size;
  for (int s = 0; s < sp_size; ++s) sc.dst[s] = o_dst[s];
  return launch_attn_tc({qkv, 3 * Dl, 0}, {qkv, 3 * Dl, Dl}, {qkv, 3 * Dl, 2 * Dl}, nullptr, D, sp_rank * Dl, B,
                        cfg->heads / sp_size, L, L, as_stream(stream), &sc);
}

int wan_sp_out_fwd(const wan_dit_config* cfg, int sp_size, const void* o, const wan_block_weights* w,
                   const float* e, float* x_inout, int B, int L, void* stream) {
  WAN_TRY(check_cfg(cfg, true));
  if (cfg->dtype != WAN_BF16) return WAN_ERR_UNSUPPORTED;
  WAN_REQUIRE(sp_size >= 1 && sp_size <= kMaxSeqRanks && L % sp_size == 0 && B >= 0 && L >= 0, WAN_ERR_SHAPE);
  WAN_REQUIRE(w, WAN_ERR_NULL);
  WAN_TRY(check_ptr(w->w_o));
  WAN_TRY(check_opt_ptr(w->b_o));
  WAN_TRY(check_opt_ptr(w->mod_bias));
  WAN_TRY(check_ptr(o));
  WAN_TRY(check_ptr(e));
  WAN_TRY(check_ptr(x_inout));
  const int D = cfg->dim, Ll = L / sp_size;
  if (B == 0 || L == 0) return WAN_OK;
  const float* gb = w->mod_bias ? w->mod_bias + 2 * D : nullptr;
  return gemm(cfg, o, D, w->w_o, w->b_o, x_inout, B * Ll, D, D, 0, epi_residual(D, e + 2 * D, gb, 6 * D, Ll),
              as_stream(stream));
}


int wan_fp8_quantize_rows(const wan_dit_config* cfg, const void* x, int M, int K, void* q, float* scale,
                          void* stream) {
  WAN_TRY(check_cfg(cfg));
  WAN_TRY(check_ptr(x));
  WAN_TRY(check_ptr(q));
  WAN_TRY(check_ptr_any(scale));
  WAN_REQUIRE(M >= 0 && K > 0 && K % 16 == 0, WAN_ERR_SHAPE);
  return launch_quantize_rows(x, K, M, K, false, q, scale, cfg->dtype, as_stream(stream));
}

int wan_fp8_quantize_tensor(const wan_dit_config* cfg, const void* x, int64_t n, void* q, float* scale,
                            void* stream) {
  WAN_TRY(check_cfg(cfg));
  WAN_TRY(check_ptr(x));
  WAN_TRY(check_ptr(q));
  WAN_TRY(check_ptr_any(scale));
  WAN_REQUIRE(n > 0 && n % 16 == 0, WAN_ERR_SHAPE);
  return launch_quantize_tensor(x, n, q, scale, cfg->dtype, as_stream(stream));
}

int wan_linear_fp8_fwd(const wan_dit_config* cfg, const void* A, const float* a_scale, const void* W,
                       const float* w_scale, const void* bias, void* out, int M, int N, int K, int epilogue,
                       const float* gate, const float* gate_bias, int64_t gate_batch_stride, int rows_per_batch,
                       void* stream) {
  WAN_TRY(check_cfg(cfg));
  if (cfg->dtype != WAN_BF16) return WAN_ERR_UNSUPPORTED;
  WAN_TRY(check_ptr(A));
  WAN_TRY(check_ptr(W));
  WAN_TRY(check_ptr_any(a_scale));
  WAN_TRY(check_ptr_any(w_scale));
  WAN_TRY(check_opt_ptr(bias));
  WAN_TRY(check_ptr(out));
  WAN_TRY(check_opt_ptr(gate));
  WAN_TRY(check_opt_ptr(gate_bias));
  WAN_REQUIRE(M >= 0 && N > 0 && K > 0 && N % 8 == 0 && K % 16 == 0, WAN_ERR_SHAPE);
  WAN_REQUIRE(epilogue >= WAN_EPI_STORE && epilogue <= WAN_EPI_F32, WAN_ERR_SHAPE);
  if (epilogue == WAN_EPI_RESIDUAL)
    WAN_REQUIRE(rows_per_batch > 0 && gate_batch_stride >= 0 && gate_batch_stride % 4 == 0, WAN_ERR_SHAPE);
  GemmEpi ep = epilogue == WAN_EPI_RESIDUAL ? epi_residual(N, gate, gate_bias, gate_batch_stride, rows_per_batch)
                                            : epi_store(N, epilogue);
  return e4m3_gemm(A, a_scale, W, w_scale, bias, out, M, N, K, ep, as_stream(stream));
}

size_t wan_fp8_workspace_bytes(const wan_dit_config* cfg, int B, int L, int Lc, int Li) {
  if (check_cfg(cfg) != WAN_OK || B < 0 || L < 0 || Lc < 0 || Li < 0) return 0;
  return fp8_layout(cfg, B, L, Lc, Li).total;
}


int wan_dit_block_fp8_fwd(const wan_dit_config* cfg, float* x, const float* e, const void* ctx, int Lc,
                          const void* img_ctx, int Li, const wan_block_weights* w, const wan_fp8_scales* sc, int B,
                          int L, void* workspace, size_t ws_bytes, void* stream) {
  WAN_TRY(check_cfg(cfg, true));
  if (cfg->dtype != WAN_BF16) return WAN_ERR_UNSUPPORTED;
  const bool with_img = img_ctx && Li > 0;
  WAN_TRY(check_block_w(cfg, w, with_img));
  WAN_TRY(check_scales(sc, with_img));
  WAN_TRY(check_ptr(x));
  WAN_TRY(check_ptr(e));
  WAN_TRY(check_ptr(ctx));
  WAN_TRY(check_opt_ptr(img_ctx));
  WAN_REQUIRE(Lc > 0 && cfg->dim % 16 == 0 && cfg->ffn_dim % 16 == 0, WAN_ERR_SHAPE);
  const int li = with_img ? Li : 0;
  WAN_TRY(check_tokens(cfg, B, L, Lc, li));
  WAN_TRY(check_ptr(workspace));
  const Fp8Layout fl = fp8_layout(cfg, B, L, Lc, li);
  WAN_REQUIRE(ws_bytes >= fl.total, WAN_ERR_WORKSPACE);
  if (B == 0 || L == 0) return WAN_OK;
  return block_fp8_impl(cfg, x, e, ctx, Lc, img_ctx, li, w, sc, B, L, workspace, fl, as_stream(stream));
}

int wan_dit_stack_fp8_fwd(const wan_dit_config* cfg, int n_blocks, const void* latent, int B, int F, int H, int W,
                          const float* t, const wan_stack_weights* sw, const wan_block_weights* blocks,
                          const wan_fp8_scales* scales, const void* ctx, int Lc, const void* img_ctx, int Li,
                          float* v_out, void* workspace, size_t ws_bytes, void* stream) {
  WAN_TRY(check_cfg(cfg, true));
  if (cfg->dtype != WAN_BF16) return WAN_ERR_UNSUPPORTED;
  WAN_REQUIRE(sw && (n_blocks == 0 || (blocks && scales)), WAN_ERR_NULL);
  WAN_REQUIRE(n_blocks >= 0 && B >= 0 && F >= 1 && H >= 2 && W >= 2 && H % 2 == 0 && W % 2 == 0, WAN_ERR_SHAPE);
  WAN_REQUIRE(Lc > 0 && cfg->dim % 16 == 0 && cfg->ffn_dim % 16 == 0, WAN_ERR_SHAPE);
  const bool with_img = img_ctx && Li > 0;
  for (int i = 0; i < n_blocks; ++i) {
    WAN_TRY(check_block_w(cfg, &blocks[i], with_img));
    WAN_TRY(check_scales(&scales[i], with_img));
  }
  WAN_TRY(check_ptr(latent));
  WAN_TRY(check_ptr(t));
  WAN_TRY(check_ptr(ctx));
  WAN_TRY(check_opt_ptr(img_ctx));
  WAN_TRY(check_ptr(v_out));
  WAN_TRY(check_ptr(sw->w_p));
  WAN_TRY(check_opt_ptr(sw->b_p));
  WAN_TRY(check_ptr(sw->w_head));
  WAN_TRY(check_opt_ptr(sw->b_head));
  WAN_TRY(check_ptr(sw->time.w_t1));
  WAN_TRY(check_ptr(sw->time.w_t2));
  WAN_TRY(check_ptr(sw->time.b_t1));
  WAN_TRY(check_ptr(sw->time.b_t2));
  WAN_TRY(check_ptr(workspace));
  const int L = F * (H / 2) * (W / 2);
  const int li = with_img ? Li : 0;
  WAN_TRY(check_tokens(cfg, B, L, Lc, li));
  const Fp8Layout fl = fp8_layout(cfg, B, L, Lc, li);
  WAN_REQUIRE(ws_bytes >= fl.total, WAN_ERR_WORKSPACE);
  if (B == 0) return WAN_OK;
  return stack_impl(cfg, n_blocks, latent, B, F, H, W, t, sw, blocks, ctx, Lc, with_img ? img_ctx : nullptr, li, v_out,
                    workspace, fl.base, as_stream(stream), nullptr, nullptr, nullptr, false, scales, &fl);
}

size_t wan_sample_workspace_bytes(const wan_dit_config* cfg, int n_blocks, int B, int F, int H, int W, int Lc,
                                  int Li, const wan_diffusion_cache* cache, int fp8) {
  if (check_cfg(cfg) != WAN_OK || n_blocks < 0 || B < 0 || F < 0 || H < 0 || W < 0 || Lc < 0 || Li < 0) return 0;
  return sample_layout(cfg, n_blocks, B, F, H, W, Lc, Li, cache != nullptr, fp8 != 0).total;
}

int wan_sample_euler_cfg(const wan_dit_config* cfg, int n_blocks, const void* input, int B, int F, int H, int W,
                         int n_steps, float guidance, const wan_stack_weights* sw, const wan_block_weights* blocks,
                         const void* ctx_cond, const void* ctx_uncond, int Lc, const void* img_ctx, int Li,
                         const wan_diffusion_cache* cache, const wan_fp8_scales* fp8_scales, float* latent_out,
                         void* workspace, size_t ws_bytes, void* stream) {
  WAN_TRY(check_cfg(cfg, true));
  WAN_REQUIRE(sw && (blocks || n_blocks == 0), WAN_ERR_NULL);
  const bool fp8 = fp8_scales != nullptr;
  if (fp8) {
    if (cfg->dtype != WAN_BF16) return WAN_ERR_UNSUPPORTED;
    WAN_REQUIRE(cfg->dim % 16 == 0 && cfg->ffn_dim % 16 == 0, WAN_ERR_SHAPE);
  }
  if (cache)
    WAN_REQUIRE(cache->attn_start >= 0 && cache->attn_interval >= 1 && cache->cfg_start >= 0 &&
                    cache->cfg_interval >= 1,
                WAN_ERR_SHAPE);
  WAN_REQUIRE(n_blocks >= 0 && n_steps >= 1 && guidance == guidance && guidance - guidance == 0.0f, WAN_ERR_SHAPE);
  WAN_REQUIRE(B >= 0 && F >= 1 && H >= 2 && W >= 2 && H % 2 == 0 && W % 2 == 0, WAN_ERR_SHAPE);
  WAN_REQUIRE(cfg->out_ch <= cfg->in_ch && Lc > 0, WAN_ERR_SHAPE);
  const bool with_img = img_ctx && Li > 0;
  for (int i = 0; i < n_blocks; ++i) {
    WAN_TRY(check_block_w(cfg, &blocks[i], with_img));
    if (fp8) WAN_TRY(check_scales(&fp8_scales[i], with_img));
  }
  WAN_TRY(check_ptr(input));
  WAN_TRY(check_ptr(ctx_cond));
  WAN_TRY(check_ptr(ctx_uncond));
  WAN_TRY(check_opt_ptr(img_ctx));
  WAN_TRY(check_ptr(latent_out));
  WAN_TRY(check_ptr(sw->w_p));
  WAN_TRY(check_opt_ptr(sw->b_p));
  WAN_TRY(check_ptr(sw->w_head));
  WAN_TRY(check_opt_ptr(sw->b_head));
  WAN_TRY(check_ptr(sw->time.w_t1));
  WAN_TRY(check_ptr(sw->time.w_t2));
  WAN_TRY(check_ptr(sw->time.b_t1));
  WAN_TRY(check_ptr(sw->time.b_t2));
  WAN_TRY(check_ptr(workspace));
  const int L = F * (H / 2) * (W / 2);
  const int li = with_img ? Li : 0;
  WAN_TRY(check_tokens(cfg, 2 * B, L, Lc, li));
  const SampleLayout sl = sample_layout(cfg, n_blocks, B, F, H, W, Lc, li, cache != nullptr, fp8);
  WAN_REQUIRE(ws_bytes >= sl.total, WAN_ERR_WORKSPACE);
  if (B == 0) return WAN_OK;
  cudaStream_t s = as_stream(stream);
  const int D = cfg->dim;
  const size_t es = dtype_size(cfg->dtype);
  const int64_t fhw = static_cast<int64_t>(F) * H * W;
  const int64_t n = cfg->out_ch * fhw, in_stride = cfg->in_ch * fhw;
  void* in2 = at(workspace, sl.in2);
  float* v = reinterpret_cast<float*>(at(workspace, sl.v));
  float* t = reinterpret_cast<float*>(at(workspace, sl.t));
  WAN_TRY(launch_sampler_init(input, B, n, in_stride, latent_out, in2, t, cfg->dtype, s));
  // Cross-attention K|V of both contexts, once per block for all steps (E4M3 projections
  // on the FP8 path, the context quantised per row in the stack workspace's code area).
  const Fp8Layout fl = fp8_layout(cfg, 2 * B, L, Lc, li);
  auto kv_proj = [&](const void* src, int rows, const void* wk, const void* bk, const float* wsc, void* dst) -> int {
    if (!fp8) return gemm(cfg, src, D, wk, bk, dst, rows, 2 * D, D, 0, epi_store(2 * D), s);
    void* codes = at(workspace, fl.ctx_codes);
    float* scl = reinterpret_cast<float*>(at(workspace, fl.ctx_scales));
    WAN_TRY(launch_quantize_rows(src, D, rows, D, false, codes, scl, WAN_BF16, s));
    return e4m3_gemm(codes, scl, wk, wsc, bk, dst, rows, 2 * D, D, epi_store(2 * D), s);
  };
  std::vector<const void*> kvt(n_blocks), kvi(n_blocks, nullptr);
  for (int i = 0; i < n_blocks; ++i) {
    uint8_t* ct = at(workspace, sl.kvt + i * sl.kvt_block);
    const size_t half_t = static_cast<size_t>(B) * Lc * 2 * D * es;
    const float* s_ckv = fp8 ? fp8_scales[i].ckv : nullptr;
    WAN_TRY(kv_proj(ctx_cond, B * Lc, blocks[i].w_ckv, blocks[i].b_ckv, s_ckv, ct));
    WAN_TRY(kv_proj(ctx_uncond, B * Lc, blocks[i].w_ckv, blocks[i].b_ckv, s_ckv, ct + half_t));
    kvt[i] = ct;
    if (with_img) {
      uint8_t* ci = at(workspace, sl.kvi + i * sl.kvi_block);
      const size_t half_i = static_cast<size_t>(B) * li * 2 * D * es;
      for (int h = 0; h < 2; ++h)
        WAN_TRY(kv_proj(img_ctx, B * li, blocks[i].w_ckv_img, blocks[i].b_ckv_img,
                        fp8 ? fp8_scales[i].ckv_img : nullptr, ci + h * half_i));
      kvi[i] = ci;
    }
  }
  // Kept attention outputs [2B, L, D] per block (conditional samples first, so a
  // conditional-only pass over B samples uses the first half) and the kept residual.
  std::vector<void*> kept;
  float* delta = nullptr;
  if (cache) {
    for (int i = 0; i < n_blocks; ++i) kept.push_back(at(workspace, sl.attn + i * sl.attn_block));
    delta = reinterpret_cast<float*>(at(workspace, sl.delta));
  }
  const Layout ly = fp8 ? fl.base : layout(cfg, 2 * B, L, Lc, li);
  const float dt = 1.0f / static_cast<float>(n_steps);
  for (int k = 0; k < n_steps; ++k) {
    bool reuse = false, skip = false;
    if (cache) {
      reuse = k >= cache->attn_start && (k - cache->attn_start) % cache->attn_interval != 0;
      skip = k >= cache->cfg_start && (k - cache->cfg_start) % cache->cfg_interval != 0;
    }
    const int Bp = skip ? B : 2 * B;  // samples in this step's pass
    WAN_TRY(stack_impl(cfg, n_blocks, in2, Bp, F, H, W, t, sw, blocks, ctx_cond, Lc,
                       with_img ? img_ctx : nullptr, li, v, workspace, ly, s,
                       n_blocks ? kvt.data() : nullptr, with_img && n_blocks ? kvi.data() : nullptr,
                       cache && n_blocks ? kept.data() : nullptr, reuse, fp8 ? fp8_scales : nullptr, &fl));
    const float t_next = static_cast<float>(1000.0 * (k + 1) / n_steps);
    WAN_TRY(launch_euler_cfg(v, B, n, in_stride, dt, guidance, latent_out, in2, t, t_next, cfg->dtype, s, delta,
                             skip));
  }
  return WAN_OK;
}

int wan_head_fwd(const wan_dit_config* cfg, const float* x, int B, int F, int H, int W, const void* w_head,
                 const void* b_head, float* v_out, void* workspace, size_t ws_bytes, void* stream) {
  WAN_TRY(check_cfg(cfg));
  WAN_TRY(check_ptr(x));
  WAN_TRY(check_ptr(w_head));
  WAN_TRY(check_opt_ptr(b_head));
  WAN_TRY(check_ptr(v_out));
  WAN_TRY(check_ptr(workspace));
  WAN_REQUIRE(B >= 0 && F >= 0 && H >= 0 && W >= 0 && H % 2 == 0 && W % 2 == 0, WAN_ERR_SHAPE);
  const int L = F * (H / 2) * (W / 2);
  WAN_REQUIRE(ws_bytes >= static_cast<size_t>(B) * L * cfg->dim * dtype_size(cfg->dtype), WAN_ERR_WORKSPACE);
  return head_impl(cfg, x, B, F, H, W, w_head, b_head, v_out, workspace, as_stream(stream));
}

int wan_i2v_input(const wan_dit_config* cfg, const void* noise, const void* cond, const uint8_t* frame_keep, int B,
                  int F, int H, int W, void* out, void* stream) {
  WAN_TRY(check_cfg(cfg));
  WAN_TRY(check_ptr(noise));
  WAN_TRY(check_ptr(cond));
  WAN_REQUIRE(frame_keep, WAN_ERR_NULL);
  WAN_TRY(check_ptr(out));
  WAN_REQUIRE(B >= 0 && F >= 1 && H >= 0 && W >= 0, WAN_ERR_SHAPE);
  return launch_i2v_input(noise, cond, frame_keep, B, F, H, W, out, cfg->dtype, as_stream(stream));
}

int wan_image_context_fwd(const wan_dit_config* cfg, const void* feat, int B, int Li, const wan_image_mlp_weights* w,
                          void* img_ctx_out, void* workspace, size_t ws_bytes, void* stream) {
  WAN_TRY(check_cfg(cfg));
  WAN_REQUIRE(w, WAN_ERR_NULL);
  WAN_TRY(check_ptr(feat));
  WAN_TRY(check_ptr(w->w_1));
  WAN_TRY(check_ptr(w->w_2));
  WAN_TRY(check_ptr(w->w_3));
  WAN_TRY(check_opt_ptr(w->b_1));
  WAN_TRY(check_opt_ptr(w->b_2));
  WAN_TRY(check_opt_ptr(w->b_3));
  WAN_TRY(check_ptr(img_ctx_out));
  WAN_TRY(check_ptr(workspace));
  WAN_REQUIRE(B >= 0 && Li >= 0 && cfg->img_feat_dim > 0 && cfg->img_feat_dim % 8 == 0, WAN_ERR_SHAPE);
  const int D = cfg->dim;
  const size_t es = dtype_size(cfg->dtype);
  const size_t half = static_cast<size_t>(B) * Li * D * es;
  WAN_REQUIRE(ws_bytes >= 2 * half, WAN_ERR_WORKSPACE);
  cudaStream_t s = as_stream(stream);
  void* t1 = workspace;
  void* t2 = static_cast<uint8_t*>(workspace) + half;
  const int M = B * Li;
  WAN_TRY(gemm(cfg, feat, cfg->img_feat_dim, w->w_1, w->b_1, t1, M, D, cfg->img_feat_dim, 0,
               epi_store(D, WAN_EPI_GELU), s));
  WAN_TRY(gemm(cfg, t1, D, w->w_2, w->b_2, t2, M, D, D, 0, epi_store(D, WAN_EPI_GELU), s));
  return gemm(cfg, t2, D, w->w_3, w->b_3, img_ctx_out, M, D, D, 0, epi_store(D), s);
}

int wan_flow_matching_input(const wan_dit_config* cfg, const void* x1, const void* x0, const float* u, int B, int64_t n,
                            void* xt_out, float* t_out, void* stream) {
  WAN_TRY(check_cfg(cfg));
  WAN_TRY(check_ptr(x1));
  WAN_TRY(check_ptr(x0));
  WAN_TRY(check_ptr(u));
  WAN_TRY(check_ptr(xt_out));
  WAN_TRY(check_opt_ptr(t_out));
  WAN_REQUIRE(B >= 0 && n >= 0, WAN_ERR_SHAPE);
  return launch_flow_input(x1, x0, u, B, n, xt_out, t_out, cfg->dtype, as_stream(stream));
}

int wan_flow_matching_loss(const wan_dit_config* cfg, const float* v, const void* x1, const void* x0, int B, int64_t n,
                           float* loss_out, void* stream) {
  WAN_TRY(check_cfg(cfg));
  WAN_TRY(check_ptr(v));
  WAN_TRY(check_ptr(x1));
  WAN_TRY(check_ptr(x0));
  WAN_TRY(check_ptr(loss_out));
  WAN_REQUIRE(B >= 0 && n > 0, WAN_ERR_SHAPE);
  return launch_flow_loss(v, x1, x0, B, n, loss_out, cfg->dtype, as_stream(stream));
}

int wan_attention_fwd(const wan_dit_config* cfg, const void* q, int64_t q_row_stride, int q_col0, const void* k,
                      int64_t k_row_stride, int k_col0, const void* v, int64_t v_row_stride, int v_col0, void* o,
                      int64_t o_row_stride, int o_col0, int B, int heads, int Lq, int Lk, int head_dim,
                      void* workspace, size_t ws_bytes, void* stream) {
  WAN_TRY(check_cfg(cfg, true));
  WAN_TRY(check_ptr(q));
  WAN_TRY(check_ptr(k));
  WAN_TRY(check_ptr(v));
  WAN_TRY(check_ptr(o));
  WAN_REQUIRE(heads == cfg->heads && head_dim == cfg->head_dim, WAN_ERR_SHAPE);
  WAN_REQUIRE(B >= 0 && Lq >= 0 && Lk > 0, WAN_ERR_SHAPE);
  const int64_t need = static_cast<int64_t>(heads) * head_dim;
  WAN_REQUIRE(q_col0 >= 0 && k_col0 >= 0 && v_col0 >= 0 && o_col0 >= 0, WAN_ERR_SHAPE);
  WAN_REQUIRE(q_col0 + need <= q_row_stride && k_col0 + need <= k_row_stride && v_col0 + need <= v_row_stride &&
                  o_col0 + need <= o_row_stride,
              WAN_ERR_SHAPE);
  if (cfg->dtype == WAN_F32) WAN_REQUIRE(Lk <= 8192, WAN_ERR_SHAPE);
  if (workspace) WAN_TRY(check_ptr(workspace));
  return attention(cfg, {q, q_row_stride, q_col0}, {k, k_row_stride, k_col0}, {v, v_row_stride, v_col0}, o,
                   o_row_stride, o_col0, B, Lq, Lk, as_stream(stream), workspace, workspace ? ws_bytes : 0);
}

size_t wan_attention_workspace_bytes(const wan_dit_config* cfg, int B, int Lq) {
  if (check_cfg(cfg) != WAN_OK || B < 0 || Lq < 0) return 0;
  return cfg->dtype == WAN_BF16 ? split_bytes(cfg, B, Lq) : 0;
}

int wan_linear_fwd(const wan_dit_config* cfg, const void* A, const void* W, const void* bias, void* out, int M, int N,
                   int K, int epilogue, const float* gate, const float* gate_bias, int64_t gate_batch_stride,
                   int rows_per_batch, void* stream) {
  WAN_TRY(check_cfg(cfg));
  WAN_TRY(check_ptr(A));
  WAN_TRY(check_ptr(W));
  WAN_TRY(check_opt_ptr(bias));
  WAN_TRY(check_ptr(out));
  WAN_TRY(check_opt_ptr(gate));
  WAN_TRY(check_opt_ptr(gate_bias));
  WAN_REQUIRE(M >= 0 && N > 0 && K > 0 && N % 8 == 0 && K % 8 == 0, WAN_ERR_SHAPE);
  WAN_REQUIRE(epilogue >= WAN_EPI_STORE && epilogue <= WAN_EPI_F32, WAN_ERR_SHAPE);
  if (epilogue == WAN_EPI_RESIDUAL) {
    WAN_REQUIRE(rows_per_batch > 0 && gate_batch_stride >= 0 && gate_batch_stride % 4 == 0, WAN_ERR_SHAPE);
  }
  GemmEpi ep = epilogue == WAN_EPI_RESIDUAL ? epi_residual(N, gate, gate_bias, gate_batch_stride, rows_per_batch)
                                            : epi_store(N, epilogue);
  return gemm(cfg, A, K, W, bias, out, M, N, K, 0, ep, as_stream(stream));
}

int check_attn_fp8_args(const wan_dit_config* cfg, const void* q, int64_t q_row_stride, int q_col0, const void* k,
                        int64_t k_row_stride, int k_col0, const void* v, int64_t v_row_stride, int v_col0, int B,
                        int heads, int Lq, int Lk, int head_dim) {
  WAN_TRY(check_cfg(cfg, true));
  if (cfg->dtype != WAN_BF16) return WAN_ERR_UNSUPPORTED;
  WAN_TRY(check_ptr(q));
  WAN_TRY(check_ptr(k));
  WAN_TRY(check_ptr(v));
  WAN_REQUIRE(heads == cfg->heads && head_dim == cfg->head_dim, WAN_ERR_SHAPE);
  WAN_REQUIRE(B >= 0 && Lq >= 0 && Lk > 0, WAN_ERR_SHAPE);
  const int64_t need = static_cast<int64_t>(heads) * head_dim;
  WAN_REQUIRE(q_col0 >= 0 && k_col0 >= 0 && v_col0 >= 0, WAN_ERR_SHAPE);
  WAN_REQUIRE(q_col0 + need <= q_row_stride && k_col0 + need <= k_row_stride && v_col0 + need <= v_row_stride,
              WAN_ERR_SHAPE);
  return WAN_OK;
}

int wan_attention_fp8_quantize(const wan_dit_config* cfg, const void* q, int64_t q_row_stride, int q_col0,
                               const void* k, int64_t k_row_stride, int k_col0, const void* v, int64_t v_row_stride,
                               int v_col0, int B, int heads, int Lq, int Lk, int head_dim, void* q_codes,
                               float* q_scale, void* k_codes, void* vt_codes, int64_t vt_stride, float* kv_scale,
                               void* stream) {
  WAN_TRY(check_attn_fp8_args(cfg, q, q_row_stride, q_col0, k, k_row_stride, k_col0, v, v_row_stride, v_col0, B,
                              heads, Lq, Lk, head_dim));
  WAN_TRY(check_ptr_any(q_codes));
  WAN_TRY(check_ptr_any(q_scale));
  WAN_TRY(check_ptr(k_codes));
  WAN_TRY(check_ptr(vt_codes));
  WAN_TRY(check_ptr_any(kv_scale));
  WAN_REQUIRE(vt_stride >= Lk && vt_stride % 64 == 0, WAN_ERR_SHAPE);
  return launch_attn_fp8_quantize(q, q_row_stride, q_col0, k, k_row_stride, k_col0, v, v_row_stride, v_col0, B, heads,
                                  Lq, Lk, q_codes, q_scale, k_codes, vt_codes, vt_stride, kv_scale,
                                  as_stream(stream));
}

int wan_attention_fp8_fwd(const wan_dit_config* cfg, const void* q, int64_t q_row_stride, int q_col0, const void* k,
                          int64_t k_row_stride, int k_col0, const void* v, int64_t v_row_stride, int v_col0, void* o,
                          int64_t o_row_stride, int o_col0, int B, int heads, int Lq, int Lk, int head_dim,
                          void* workspace, size_t ws_bytes, void* stream) {
  WAN_TRY(check_attn_fp8_args(cfg, q, q_row_stride, q_col0, k, k_row_stride, k_col0, v, v_row_stride, v_col0, B,
                              heads, Lq, Lk, head_dim));
  WAN_TRY(check_ptr(o));
  WAN_REQUIRE(o_col0 >= 0 && o_col0 + static_cast<int64_t>(heads) * head_dim <= o_row_stride, WAN_ERR_SHAPE);
  WAN_TRY(check_ptr(workspace));
  const AttnF8Layout l = attn_f8_layout(cfg, B, Lq, Lk);
  WAN_REQUIRE(ws_bytes >= l.total, WAN_ERR_WORKSPACE);
  if (B == 0 || Lq == 0) return WAN_OK;
  uint8_t* w = static_cast<uint8_t*>(workspace);
  float* qs = reinterpret_cast<float*>(w + l.qs);
  float* kvs = reinterpret_cast<float*>(w + l.kvs);
  cudaStream_t s = as_stream(stream);
  WAN_TRY(launch_attn_fp8_quantize(q, q_row_stride, q_col0, k, k_row_stride, k_col0, v, v_row_stride, v_col0, B,
                                   heads, Lq, Lk, w + l.qc, qs, w + l.kc, w + l.vt, l.vt_stride, kvs, s));
  return launch_attn_tc_fp8(w + l.qc, qs, w + l.kc, w + l.vt, l.vt_stride, kvs, o, o_row_stride, o_col0, B, heads,
                            Lq, Lk, s, w + l.split, l.split_bytes);
}

size_t wan_attention_fp8_workspace_bytes(const wan_dit_config* cfg, int B, int Lq, int Lk) {
  if (check_cfg(cfg) != WAN_OK || cfg->dtype != WAN_BF16 || B < 0 || Lq < 0 || Lk <= 0) return 0;
  return attn_f8_layout(cfg, B, Lq, Lk).total;
}

int64_t wan_launch_count(void) { return g_launches.load(); }

int wan_trace_enable(int on) {
  Trace& t = trace();
  std::lock_guard<std::mutex> lk(t.mu);
  if (on && t.start.empty()) {
    t.start.resize(kTracePairs);
    t.stop.resize(kTracePairs);
    t.kind.assign(kTracePairs, -1);
    t.work.assign(kTracePairs, 0.0);
    for (int i = 0; i < kTracePairs; ++i) {
      if (cudaEventCreate(&t.start[i]) != cudaSuccess || cudaEventCreate(&t.stop[i]) != cudaSuccess) {
        t.start.resize(i);
        t.stop.resize(i);
        return WAN_ERR_CUDA;
      }
    }
  }
  t.on = on != 0;
  return WAN_OK;
}

int wan_trace_reset(void) {
  Trace& t = trace();
  std::lock_guard<std::mutex> lk(t.mu);
  t.used = 0;
  return WAN_OK;
}

int wan_trace_read(int kind, double* total_ms, int64_t* launches) {
  WAN_REQUIRE(total_ms && launches, WAN_ERR_NULL);
  Trace& t = trace();
  std::lock_guard<std::mutex> lk(t.mu);
  double tot = 0.0;
  int64_t n = 0;
  for (int i = 0; i < t.used; ++i) {
    if (t.kind[i] != kind) continue;
    if (cudaEventSynchronize(t.stop[i]) != cudaSuccess) return WAN_ERR_CUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, t.start[i], t.stop[i]) != cudaSuccess) return WAN_ERR_CUDA;
    tot += ms;
    ++n;
  }
  *total_ms = tot;
  *launches = n;
  return WAN_OK;
}

int wan_trace_launches(int cap, int* kinds, double* ms, double* work) {
  WAN_REQUIRE(cap >= 0 && (cap == 0 || (kinds && ms && work)), WAN_ERR_NULL);
  Trace& t = trace();
  std::lock_guard<std::mutex> lk(t.mu);
  const int n = t.used < cap ? t.used : cap;
  for (int i = 0; i < n; ++i) {
    if (cudaEventSynchronize(t.stop[i]) != cudaSuccess) return WAN_ERR_CUDA;
    float e = 0.f;
    if (cudaEventElapsedTime(&e, t.start[i], t.stop[i]) != cudaSuccess) return WAN_ERR_CUDA;
    kinds[i] = t.kind[i];
    ms[i] = e;
    work[i] = t.work[i];
  }
  return n;
}

}  // extern "C"
