/*
 * wan.h - C ABI of the B200 (sm_100a) library for the Wan 2.1 DiT forward hot path.
 *
 * The operations follow "Wan: Open and Advanced Large-Scale Video Generative Models
 * (Wan 2.1)" (zhao9797.github.io), section "Diffusion Transformer" (patchify with a
 * (1,2,2) 3D convolution, a shared Linear+SiLU timestep MLP predicting six modulation
 * vectors with a learned bias per block, full spatio-temporal self-attention, text
 * cross-attention, FFN, unpatchify), its config table (dim / FFN dim / heads / layers,
 * frequency dim 256, latent dim 16), section "I2V 架构扩展" (I2V input fusion and
 * decoupled image cross-attention) and section "训练方法" (rectified-flow
 * interpolation and velocity target).
 *
 * Conventions for every call:
 *  - Pointers to tensors are DEVICE pointers owned by the caller; the library never
 *    allocates device memory. Calls that need scratch take a caller-provided device
 *    workspace (size from wan_workspace_bytes). Struct pointers (config, weight
 *    tables) are HOST pointers read during the call only.
 *  - Tensors are dense, row-major, in the listed shapes. "act" means the activation /
 *    weight dtype of the config (cfg->dtype: WAN_F32 or WAN_BF16). The residual
 *    stream x, the modulation e and mod_bias, timesteps and outputs of patchify/head
 *    are always fp32.
 *  - Linear weights are [out_features, in_features] (y = x W^T + b), biases [out].
 *  - Every device pointer must be 16-byte aligned.
 *  - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream). Arguments are validated on the host before any launch; on a
 *    validation error nothing is launched and a negative wan_status is returned.
 *    Launch failures return WAN_ERR_CUDA. Device-side waits are bounded: a wait that
 *    runs out sets a device flag that wan_device_status() reports as WAN_ERR_TIMEOUT.
 *  - Calls keep no state between them except the trace tables and the device error
 *    flag; they are safe to call from several host threads on different streams.
 *  - Shape limits: D = heads * head_dim; head_dim 128 (bf16) or <= 128 (fp32);
 *    D, ffn_dim multiples of 64; freq_dim a multiple of 8; latent H and W even; the
 *    fp32 path supports key lengths up to 8192.
 */
#ifndef WAN_H
#define WAN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  WAN_OK = 0,
  WAN_ERR_NULL = -1,        /* a required pointer is NULL                          */
  WAN_ERR_SHAPE = -2,       /* sizes inconsistent or outside the supported range   */
  WAN_ERR_DTYPE = -3,       /* unknown dtype                                       */
  WAN_ERR_ALIGN = -4,       /* a device pointer is not 16-byte aligned             */
  WAN_ERR_WORKSPACE = -5,   /* workspace smaller than wan_workspace_bytes()        */
  WAN_ERR_CUDA = -6,        /* a CUDA launch or runtime call failed                */
  WAN_ERR_TIMEOUT = -7,     /* a bounded device-side wait ran out                  */
  WAN_ERR_UNSUPPORTED = -8  /* valid request this build does not implement         */
} wan_status;

typedef enum { WAN_F32 = 0, WAN_BF16 = 1 } wan_dtype;

/* Model hyper-parameters (config table of the Wan 2.1 page). */
typedef struct {
  int dim;          /* D: model width                       (1536 / 5120)   */
  int heads;        /* attention heads                      (12 / 40)       */
  int head_dim;     /* D / heads                            (128)           */
  int ffn_dim;      /* F: FFN hidden width                  (8960 / 13824)  */
  int in_ch;        /* DiT input channels: 16 (T2V) or 36 (I2V)             */
  int out_ch;       /* output latent channels (16)                          */
  int freq_dim;     /* sinusoidal timestep embedding width (256)            */
  int img_feat_dim; /* image-encoder feature width for I2V (1280)           */
  float eps;        /* LayerNorm epsilon (1e-6), no affine                  */
  int dtype;        /* wan_dtype of weights and activations                 */
} wan_dit_config;

/* One DiT block's weights (act dtype unless noted). */
typedef struct {
  const float* mod_bias;            /* [6, D] fp32: per-block bias added to e  */
  const void *w_qkv, *b_qkv;        /* [3D, D], [3D]: stacked q, k, v          */
  const void *w_o, *b_o;            /* [D, D], [D]                             */
  const void *w_cq, *b_cq;          /* [D, D], [D]: cross-attention query      */
  const void *w_ckv, *b_ckv;        /* [2D, D], [2D]: text key, value          */
  const void *w_co, *b_co;          /* [D, D], [D]: cross-attention output     */
  const void *w_ckv_img, *b_ckv_img;/* [2D, D], [2D]: I2V image key, value; NULL for T2V */
  const void *w_1, *b_1;            /* [F, D], [F]                             */
  const void *w_2, *b_2;            /* [D, F], [D]                             */
} wan_block_weights;

/* Shared timestep MLP: sinusoid(freq_dim) -> Linear(freq_dim, D) -> SiLU -> Linear(D, 6D). */
typedef struct {
  const void *w_t1, *b_t1;          /* [D, freq_dim], [D]   */
  const void *w_t2, *b_t2;          /* [6D, D], [6D]        */
} wan_time_weights;

/* I2V image-context MLP: Linear(img_feat, D) -> GELU -> Linear(D, D) -> GELU -> Linear(D, D). */
typedef struct {
  const void *w_1, *b_1;            /* [D, img_feat], [D] */
  const void *w_2, *b_2;            /* [D, D], [D]        */
  const void *w_3, *b_3;            /* [D, D], [D]        */
} wan_image_mlp_weights;

/* Non-block weights of the whole DiT. */
typedef struct {
  const void *w_p, *b_p;            /* patchify conv [D, in_ch, 1, 2, 2] (= [D, in_ch*4]), [D] */
  wan_time_weights time;
  const void *w_head, *b_head;      /* [out_ch*4, D], [out_ch*4]: head Linear, (c, ph, pw) order */
} wan_stack_weights;

/* Linear-layer epilogues of wan_linear_fwd (and of the block's GEMMs). */
typedef enum {
  WAN_EPI_STORE = 0,     /* out(act)  = A W^T + b                                  */
  WAN_EPI_GELU = 1,      /* out(act)  = gelu_tanh(A W^T + b)                       */
  WAN_EPI_RESIDUAL = 2,  /* out(fp32) += g * (A W^T + b), g = gate[b,n]+gate_bias[n] (1 if gate NULL) */
  WAN_EPI_F32 = 3        /* out(fp32) = A W^T + b                                  */
} wan_epilogue;

/* Trace kinds (wan_trace_read). */
typedef enum { WAN_KIND_NORM = 0, WAN_KIND_GEMM = 1, WAN_KIND_ATTN = 2, WAN_KIND_SMALL = 3,
               WAN_KIND_COUNT = 4 } wan_kernel_kind;

/* ---- library information ------------------------------------------------------- */

/* Human-readable text of a wan_status. Never NULL; static storage. */
const char* wan_status_string(int status);

/* Device-memory workspace (bytes) that wan_dit_block_fwd / wan_dit_stack_fwd and the
 * branch calls need for batch B, L video tokens, Lc text tokens and Li image tokens
 * (Li = 0 for T2V). Returns 0 for an invalid config. */
size_t wan_workspace_bytes(const wan_dit_config* cfg, int B, int L, int Lc, int Li);

/* Sync `stream`, then report and clear the device flag set by a bounded wait that ran
 * out: WAN_OK, WAN_ERR_TIMEOUT, or WAN_ERR_CUDA if the sync itself failed. */
int wan_device_status(void* stream);

/* Exercises the failure path of the kernels' bounded waits: launches one thread that
 * waits on a barrier nothing arrives at. The wait gives up after its limit (1 s) and
 * records WAN_ERR_TIMEOUT in the device flag, which the next wan_device_status returns
 * (and clears); the context stays usable. No fault, trap or hang is involved. Returns
 * WAN_OK once launched (or WAN_ERR_CUDA). */
int wan_wait_timeout_check(void* stream);

/* ---- the hot path -------------------------------------------------------------- */

/* Patchify [Wan 2.1 page, "Diffusion Transformer": 3D conv, kernel = stride = (1,2,2)].
 * latent [B, in_ch, F, H, W] act; x_out [B, L, D] fp32 with L = F*(H/2)*(W/2), tokens
 * ordered (f, i, j). Workspace: B*L*in_ch*4 act elements (the gathered patches). */
int wan_patchify(const wan_dit_config* cfg, const void* latent, int B, int F, int H, int W,
                 const void* w_p, const void* b_p, float* x_out,
                 void* workspace, size_t ws_bytes, void* stream);

/* Shared timestep MLP [Wan 2.1 page, "Diffusion Transformer"]: t [B] fp32 (0..1000
 * scale) -> e_out [B, 6, D] fp32 = Linear(D,6D)(SiLU(Linear(256,D)(sinusoid(t)))).
 * The sinusoid is [cos(t f_i) | sin(t f_i)], f_i = 10000^(-i/(freq_dim/2)). */
int wan_time_mlp(const wan_dit_config* cfg, const float* t, int B, const wan_time_weights* w,
                 float* e_out, void* stream);

/* LayerNorm (eps, no affine) + AdaLN modulation [Wan 2.1 page, "Diffusion Transformer":
 * six modulation vectors]. x [B, L, D] fp32 -> h_out [B, L, D] act with
 * h = LN(x) * (1 + scale) + shift, where for chunk c in {0, 1}
 * shift = e[b, 3c] + mod_bias[3c], scale = e[b, 3c+1] + mod_bias[3c+1]
 * (chunk 0: self-attention input, chunk 1: FFN input). chunk = -1 gives plain LN and
 * ignores e and mod_bias. mod_bias may be NULL (zero). */
int wan_adaln_modulate(const wan_dit_config* cfg, const float* x, int B, int L,
                       const float* e, const float* mod_bias, int chunk, void* h_out, void* stream);

/* Self-attention branch with gated residual [Wan 2.1 page, "Diffusion Transformer":
 * full spatio-temporal self-attention in every block, whose output is scaled by one of
 * the six modulation vectors, the gate]: x_inout[B, L, D] fp32 +=
 * gate_msa * (Attn(h Wq, h Wk, h Wv) Wo^T + bo), gate_msa = e[b,2] + w->mod_bias[2].
 * h [B, L, D] act is the modulated LN output. Attention is full (non-causal) over the
 * L tokens of each sample, per head, scale 1/sqrt(head_dim). */
int wan_self_attn_fwd(const wan_dit_config* cfg, const void* h, const wan_block_weights* w,
                      const float* e, float* x_inout, int B, int L,
                      void* workspace, size_t ws_bytes, void* stream);

/* Cross-attention branch, plain residual [Wan 2.1 page, "Diffusion Transformer" and
 * "I2V 架构扩展"]: x_inout += (Attn(q, Kt, Vt) [+ Attn(q, Ki, Vi)]) Wco^T + bco with
 * q = h Wcq^T + bcq, [Kt|Vt] = ctx Wckv^T + bckv, [Ki|Vi] = img_ctx Wckv_img^T + b.
 * h [B, L, D] act (plain LN of x); ctx [B, Lc, D] act; img_ctx [B, Li, D] act or NULL
 * (Li = 0). */
int wan_cross_attn_fwd(const wan_dit_config* cfg, const void* h, const void* ctx, int Lc,
                       const void* img_ctx, int Li, const wan_block_weights* w,
                       float* x_inout, int B, int L, void* workspace, size_t ws_bytes, void* stream);

/* FFN branch with gated residual [Wan 2.1 page, "Diffusion Transformer" and the config
 * table (FFN dimension 8960 / 13824): the block's feed-forward network, its output scaled
 * by the sixth modulation vector]: x_inout += gate_ffn * (gelu_tanh(h W1^T + b1) W2^T + b2),
 * gate_ffn = e[b,5] + w->mod_bias[5]. h [B, L, D] act. */
int wan_ffn_fwd(const wan_dit_config* cfg, const void* h, const wan_block_weights* w,
                const float* e, float* x_inout, int B, int L,
                void* workspace, size_t ws_bytes, void* stream);

/* One DiT block [Wan 2.1 page, "Diffusion Transformer": self-attention, cross-attention
 * to the text embedding, and an FFN; a shared MLP of the timestep gives six modulation
 * vectors (shift, scale and gate of two branches) and each block learns its own bias on
 * top of them], in place on the residual stream x_inout [B, L, D] fp32:
 * self-attention (modulated LN, gated), cross-attention (plain LN, ungated), FFN
 * (modulated LN, gated). e [B, 6, D] fp32 is the shared timestep-MLP output; the
 * block adds w->mod_bias. ctx [B, Lc, D] act; img_ctx [B, Li, D] act or NULL. */
int wan_dit_block_fwd(const wan_dit_config* cfg, float* x_inout, const float* e,
                      const void* ctx, int Lc, const void* img_ctx, int Li,
                      const wan_block_weights* w, int B, int L,
                      void* workspace, size_t ws_bytes, void* stream);

/* The whole DiT: patchify -> shared timestep MLP -> n_blocks blocks (blocks is a HOST
 * array of n_blocks weight tables) -> head (plain LN, Linear(D, out_ch*4)) ->
 * unpatchify. latent [B, in_ch, F, H, W] act, t [B] fp32, ctx [B, Lc, D] act,
 * img_ctx [B, Li, D] act or NULL; v_out [B, out_ch, F, H, W] fp32 (the predicted
 * velocity). Workspace: wan_workspace_bytes(...) of this L. */
int wan_dit_stack_fwd(const wan_dit_config* cfg, int n_blocks, const void* latent,
                      int B, int F, int H, int W, const float* t,
                      const wan_stack_weights* sw, const wan_block_weights* blocks,
                      const void* ctx, int Lc, const void* img_ctx, int Li,
                      float* v_out, void* workspace, size_t ws_bytes, void* stream);

/* Head and unpatchify [Wan 2.1 page, "Diffusion Transformer"]: x [B, L, D] fp32 ->
 * plain LN -> Linear(D, out_ch*4) -> v_out [B, out_ch, F, H, W] fp32, where output
 * column c*4 + ph*2 + pw of token (f, i, j) lands at v_out[b, c, f, 2i+ph, 2j+pw].
 * Workspace: B*L*D act elements. */
int wan_head_fwd(const wan_dit_config* cfg, const float* x, int B, int F, int H, int W,
                 const void* w_head, const void* b_head, float* v_out,
                 void* workspace, size_t ws_bytes, void* stream);

/* ---- patchify without a workspace --------------------------------------------- */

/* Bytes of the fixed device scratch array that wan_patchify_noalloc uses. */
#define WAN_PATCHIFY_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)

/* wan_patchify for callers that cannot allocate device memory: code that must not call
 * the CUDA allocator (a host callback, an allocation-free real-time loop), a plug-in
 * that its host framework hands only input and output pointers, or a process whose
 * device-memory budget is fixed at start-up. The Wan 2.1 pages have no counterpart of
 * this call; it exists for such callers of this library.
 * Same arguments, layout and result as wan_patchify minus the workspace: the gathered
 * patches go to a fixed array of WAN_PATCHIFY_NOALLOC_SCRATCH_BYTES (16 MiB) inside the
 * library, which every GPU that loads the library holds until the process exits. A
 * request whose patches (B*L*in_ch*4 act elements) exceed it returns WAN_ERR_SHAPE
 * before any launch. The call allocates nothing (no cudaMalloc, no cudaFree, no
 * allocating library routine).
 * The first call on a device looks up the array's device address (with that device
 * current) and caches it; make that first call before any stream capture. The cached
 * address belongs to the CUDA context it was looked up in: after a device reset, the
 * next call on that device looks it up again, so make that call, too, before any
 * capture. All calls
 * share the one array and each leaves its contents behind: calls whose work overlaps
 * on the GPU (other streams, other host threads) race on it, so the caller must order
 * them. No part of the array needs to start at zero. */
int wan_patchify_noalloc(const wan_dit_config* cfg, const void* latent, int B, int F, int H, int W,
                         const void* w_p, const void* b_p, float* x_out, void* stream);

/* ---- I2V and flow-matching pieces --------------------------------------------- */

/* I2V input fusion [Wan 2.1 page, "I2V 架构扩展"]: out [B, 36, F, H, W] act =
 * concat(noise [B,16,F,H,W], cond [B,16,F,H,W], mask [B,4,F,H,W]) where the mask is
 * built from frame_keep [B, 1+4(F-1)] uint8 (1 = keep, 0 = generate): the first
 * frame's value is repeated 4 times, the 4F values are grouped per latent frame and
 * put on 4 channels, broadcast over H x W. */
int wan_i2v_input(const wan_dit_config* cfg, const void* noise, const void* cond,
                  const uint8_t* frame_keep, int B, int F, int H, int W, void* out, void* stream);

/* I2V image-context MLP: feat [B, Li, img_feat] act -> img_ctx_out [B, Li, D] act.
 * Workspace: 2 * B * Li * D act elements. */
int wan_image_context_fwd(const wan_dit_config* cfg, const void* feat, int B, int Li,
                          const wan_image_mlp_weights* w, void* img_ctx_out,
                          void* workspace, size_t ws_bytes, void* stream);

/* Rectified-flow interpolation [Wan 2.1 page, "训练方法"]: xt_out[b] = u[b] x1[b] +
 * (1 - u[b]) x0[b] (act, n elements per sample), and t_out[b] = 1000 u[b] (fp32). */
int wan_flow_matching_input(const wan_dit_config* cfg, const void* x1, const void* x0,
                            const float* u, int B, int64_t n, void* xt_out, float* t_out,
                            void* stream);

/* Mean squared error per sample between the prediction v [B, n] fp32 and the
 * velocity target x1 - x0 (act): loss_out [B] fp32. */
int wan_flow_matching_loss(const wan_dit_config* cfg, const float* v, const void* x1,
                           const void* x0, int B, int64_t n, float* loss_out, void* stream);

/* ---- FP8 (E4M3) linear layers ------------------------------------------------- */

/* FP8 GEMMs as the pages describe for inference [Wan 2.1 page, "Infra", inference
 * optimisation: FP8 GEMM with a per-tensor scale for the weights and a per-token scale
 * for the activations]. Codes are E4M3 (OCP FP8: bias 7, subnormals, no infinities),
 * q = round-to-nearest-even-satfinite(x / s), s = amax / 448 (1 for an all-zero row or
 * tensor), computed in IEEE float32. Requires a bf16 config; E4M3 arrays are bytes. */

/* Per-tensor scales (device fp32 scalars) of a block's E4M3 weights. ckv_img may be
 * NULL for T2V. attention_fp8 nonzero: the block's self-attention also runs on E4M3
 * operands (the 8-bit attention of wan_attention_fp8_fwd, below); the text and image
 * cross-attention stay bf16 (with 512 or 257 keys, quantising their queries costs more
 * than the 8-bit products save). */
typedef struct {
  const float *qkv, *o, *cq, *ckv, *co, *ckv_img, *ffn1, *ffn2;
  int attention_fp8;
} wan_fp8_scales;

/* Codes of x [M, K] act, one scale per row: q [M, K] E4M3, scale [M] fp32 (device).
 * K % 16 == 0. */
int wan_fp8_quantize_rows(const wan_dit_config* cfg, const void* x, int M, int K, void* q, float* scale,
                          void* stream);

/* Codes of a whole tensor x [n] act with one scale: q [n] E4M3, scale[0] fp32 (device;
 * it is used as scratch while the work runs). n % 16 == 0. For weights, once. */
int wan_fp8_quantize_tensor(const wan_dit_config* cfg, const void* x, int64_t n, void* q, float* scale,
                            void* stream);

/* y = a_scale[m] * w_scale[0] * (A W^T) + bias, then the epilogue of wan_linear_fwd.
 * A [M, K] E4M3 (row stride K), a_scale [M] fp32, W [N, K] E4M3, w_scale [1] fp32,
 * bias [N] act or NULL. K % 16 == 0, N % 8 == 0. tcgen05 kind::f8f6f4. */
int wan_linear_fp8_fwd(const wan_dit_config* cfg, const void* A, const float* a_scale, const void* W,
                       const float* w_scale, const void* bias, void* out, int M, int N, int K, int epilogue,
                       const float* gate, const float* gate_bias, int64_t gate_batch_stride,
                       int rows_per_batch, void* stream);

/* Workspace (bytes) of wan_dit_block_fp8_fwd: the bf16 block's workspace, the E4M3 codes
 * and row scales of the activations and the context, and the operands of the 8-bit
 * self-attention (used only with attention_fp8; about 3 B*L*dim bytes). */
size_t wan_fp8_workspace_bytes(const wan_dit_config* cfg, int B, int L, int Lc, int Li);

/* wan_dit_block_fwd with every linear layer in FP8: w holds E4M3 codes for the eight
 * weight matrices (biases and mod_bias as in the bf16 call) and sc their scales. The
 * LayerNorm kernels write E4M3 codes with per-row scales directly; the attention
 * outputs, the context, the image context and the FFN hidden are quantised per row by
 * a separate pass (the I2V text and image attention outputs are summed first).
 * Attention itself stays bf16 with fp32 accumulation. D % 16 == 0, F % 16 == 0, and
 * D in {512, 1536, 5120} (WAN_ERR_UNSUPPORTED else). */
int wan_dit_block_fp8_fwd(const wan_dit_config* cfg, float* x_inout, const float* e, const void* ctx, int Lc,
                          const void* img_ctx, int Li, const wan_block_weights* w, const wan_fp8_scales* sc,
                          int B, int L, void* workspace, size_t ws_bytes, void* stream);

/* wan_dit_stack_fwd with every block as in wan_dit_block_fp8_fwd: blocks hold E4M3 codes
 * and scales is a HOST array of n_blocks weight-scale tables; patchify, the timestep
 * MLP and the head stay bf16. Workspace: wan_fp8_workspace_bytes(cfg, B, L, Lc, Li). */
int wan_dit_stack_fp8_fwd(const wan_dit_config* cfg, int n_blocks, const void* latent, int B, int F, int H,
                          int W, const float* t, const wan_stack_weights* sw,
                          const wan_block_weights* blocks, const wan_fp8_scales* scales, const void* ctx,
                          int Lc, const void* img_ctx, int Li, float* v_out, void* workspace,
                          size_t ws_bytes, void* stream);

/* ---- sequence parallelism (Ulysses) ------------------------------------------ */

/* Self-attention of one block split over P = sp_size ranks along the token axis, the
 * intra-machine layer of the pages' context parallelism [163.com article on Wan2.1,
 * "核心创新三" (inference: context parallelism; inside a machine, Ulysses); Wan 2.1 page,
 * "Infra" (2D CP = outer Ring Attention x inner Ulysses)]. Rank r owns tokens
 * [r L/P, (r+1) L/P) of every sample, and heads [r H/P, (r+1) H/P) while attending.
 * Everything except attention is row-local and uses the ordinary calls on L/P rows.
 * The exchange is fused into the producing kernels: each call stores its results
 * straight into the buffers of the ranks that consume them (pointers that may be peer
 * GPUs' memory, e.g. CUDA IPC mappings over NVLink; on one GPU, local buffers). The
 * caller orders the phases across ranks (all ranks finish phase 1 before any starts
 * phase 2, and so on), e.g. with a one-element all-reduce on the stream.
 * Requirements: bf16 config (WAN_ERR_UNSUPPORTED otherwise), 1 <= P <= 8, H % P == 0,
 * L % P == 0, 0 <= sp_rank < P; pointer arrays are HOST arrays of P device pointers,
 * each 16-byte aligned. Errors are returned before any launch. */

/* Phase 1 - QKV projection and scatter: h [B, L/P, D] act (this rank's rows of the
 * modulated LN output). Computes h Wqkv^T + b and stores, for every rank s, the q, k and
 * v columns of s's heads into qkv_dst[s] [B, L, 3D/P] act (q | k | v slabs of D/P
 * columns) at this rank's rows. */
int wan_sp_qkv_fwd(const wan_dit_config* cfg, int sp_size, int sp_rank, const void* h, int B, int L,
                   const wan_block_weights* w, void* const* qkv_dst, void* stream);

/* Phase 2 - attention and gather: qkv [B, L, 3D/P] act (this rank's heads, all rows, as
 * phase 1 left it). Attends over all L tokens and stores each row's output of this
 * rank's heads into o_dst[owner] [B, L/P, D] act, columns [sp_rank D/P, (sp_rank+1) D/P),
 * where owner = row / (L/P). */
int wan_sp_attn_fwd(const wan_dit_config* cfg, int sp_size, int sp_rank, const void* qkv, int B, int L,
                    void* const* o_dst, void* stream);

/* Phase 3 - output projection with the gated residual on this rank's rows:
 * x_inout [B, L/P, D] fp32 += gate_msa * (o Wo^T + bo), o [B, L/P, D] act from phase 2,
 * gate_msa = e[b, 2] + w->mod_bias[2] (e [B, 6, D] fp32). */
int wan_sp_out_fwd(const wan_dit_config* cfg, int sp_size, const void* o, const wan_block_weights* w,
                   const float* e, float* x_inout, int B, int L, void* stream);

/* ---- sampling ----------------------------------------------------------------- */

/* Diffusion cache of the sampling loop [Wan 2.1 page, "Infra", inference optimisation:
 * a block's attention output changes little between steps and is computed every few
 * steps; late steps skip the unconditional pass and correct the conditional prediction
 * by a kept residual]. Step k reuses every block's attention output when
 * k >= attn_start and (k - attn_start) % attn_interval != 0, and skips the
 * unconditional pass when k >= cfg_start and (k - cfg_start) % cfg_interval != 0.
 * Intervals >= 1 (1 = never); starts >= 0; step 0 always runs both passes in full. On a
 * skipped step the guided velocity is v_c + (guidance - 1) delta, delta = v_c - v_u
 * from the last step that ran both passes. Each pass keeps its own attention outputs
 * (those of the last step on which that pass computed attention). */
typedef struct {
  int attn_start, attn_interval;
  int cfg_start, cfg_interval;
} wan_diffusion_cache;

/* Device workspace (bytes) of wan_sample_euler_cfg for these sizes, cache (NULL = no
 * cache) and precision (fp8 != 0: FP8 linear layers); 0 on a bad cfg. The cache adds
 * n_blocks x 2B x L x D act elements of kept attention outputs and
 * B x out_ch x F x H x W fp32 of kept residual. */
size_t wan_sample_workspace_bytes(const wan_dit_config* cfg, int n_blocks, int B, int F, int H, int W,
                                  int Lc, int Li, const wan_diffusion_cache* cache, int fp8);

/* Generation loop with the DiT as the velocity model [Wan 2.1 page, "训练方法" (the
 * rectified-flow velocity) and "Infra" (a fixed number of sampling steps, about 50); the
 * Baidu cloud article on Wan 2.1 names the step count and the guidance scale as the
 * user's knobs]. The pages fix neither the time grid nor the solver nor the guidance
 * formula; this call takes the plainest reading that the velocity definition supports:
 * x(0) is the noise, x(1) the sample, n_steps explicit Euler steps on the uniform grid
 * t_k = k / n_steps, x += (1/n_steps) (v_u + guidance (v_c - v_u)), where
 * v_c = DiT(input(x), 1000 t_k, ctx_cond) and v_u = DiT(input(x), 1000 t_k, ctx_uncond)
 * are evaluated as ONE stack pass over a batch of 2B samples.
 *   input [B, in_ch, F, H, W] act (device): the noise in channels [0, out_ch) and, for
 *     I2V (in_ch > out_ch), the condition channels [out_ch, in_ch) that are appended to
 *     x unchanged at every step. out_ch <= in_ch.
 *   ctx_cond, ctx_uncond [B, Lc, D] act; img_ctx [B, Li, D] act or NULL (Li = 0): the
 *     image context is shared by both branches.
 *   latent_out [B, out_ch, F, H, W] fp32: the state x, written with the noise at the
 *     start and holding x(1) on return. The DiT input is x rounded to act each step.
 *   blocks: HOST array of n_blocks weight tables; sw: stack weights.
 *   Cross-attention K|V of both contexts are projected once per call and kept for all
 *   steps. cache: NULL (every step runs both passes in full) or the diffusion cache
 *   above. fp8_scales: NULL (bf16 linear layers) or, with blocks holding E4M3 codes,
 *   a HOST array of n_blocks weight-scale tables: every block runs as in
 *   wan_dit_block_fp8_fwd (the K|V projections of the contexts too).
 *   workspace >= wan_sample_workspace_bytes(...) device bytes (same cache, fp8).
 * Errors (before any launch): WAN_ERR_NULL, WAN_ERR_SHAPE (n_steps < 1, a guidance that
 * is not finite, out_ch > in_ch, Lc = 0, odd H or W, a cache interval < 1 or start < 0),
 * WAN_ERR_WORKSPACE, WAN_ERR_ALIGN.
 * B = 0 returns WAN_OK without work. Enqueued on `stream`; returns before the GPU work
 * ends. */
int wan_sample_euler_cfg(const wan_dit_config* cfg, int n_blocks, const void* input, int B, int F, int H,
                         int W, int n_steps, float guidance, const wan_stack_weights* sw,
                         const wan_block_weights* blocks, const void* ctx_cond, const void* ctx_uncond,
                         int Lc, const void* img_ctx, int Li, const wan_diffusion_cache* cache,
                         const wan_fp8_scales* fp8_scales, float* latent_out, void* workspace,
                         size_t ws_bytes, void* stream);

/* ---- single-kernel entry points (used by the branch calls; exposed for tests) --- */

/* Multi-head attention softmax(q k^T / sqrt(d)) v, non-causal. q [B, Lq, *], k and v
 * [B, Lk, *], o [B, Lq, *] act; head h of each operand occupies columns
 * [col0 + h*d, col0 + (h+1)*d) of rows with the given row strides (elements).
 * workspace (optional, device, NULL with ws_bytes 0): with at least
 * wan_attention_workspace_bytes(...) bytes, a last wave of work units that would fill
 * at most half of the SMs is split over the key tiles and merged (bf16 path). */
int wan_attention_fwd(const wan_dit_config* cfg, const void* q, int64_t q_row_stride, int q_col0,
                      const void* k, int64_t k_row_stride, int k_col0,
                      const void* v, int64_t v_row_stride, int v_col0,
                      void* o, int64_t o_row_stride, int o_col0,
                      int B, int heads, int Lq, int Lk, int head_dim, void* workspace, size_t ws_bytes,
                      void* stream);

/* Bytes of the optional wan_attention_fwd workspace for B samples of Lq queries. */
size_t wan_attention_workspace_bytes(const wan_dit_config* cfg, int B, int Lq);

/* y = A W^T + b with an epilogue. A [M, K] act (row stride K), W [N, K] act, bias [N]
 * act or NULL. out: act [M, N] for STORE/GELU, fp32 [M, N] for F32/RESIDUAL. For
 * RESIDUAL, gate (fp32) is indexed gate[(m / rows_per_batch) * gate_batch_stride + n]
 * and gate_bias [N] fp32 is added (either may be NULL). */
int wan_linear_fwd(const wan_dit_config* cfg, const void* A, const void* W, const void* bias,
                   void* out, int M, int N, int K, int epilogue,
                   const float* gate, const float* gate_bias, int64_t gate_batch_stride,
                   int rows_per_batch, void* stream);

/* ---- 8-bit attention --------------------------------------------------------------- */

/* 8-bit attention [Wan 2.1 page, "Infra", inference optimisation: 8-bit FlashAttention,
 * INT8 for q k^T and FP8 for the product with v], here with E4M3 for both products
 * (the tensor cores' f8 kind; tcgen05 kind::f8f6f4). Scales (each amax / 448 as above,
 * IEEE float32): q per (sample, token, head); k and v per (sample, head) over all key
 * rows. The probabilities p = 2^(s log2e / sqrt(d) - base) are rounded to E4M3 for the
 * product with v; the normaliser is the fp32 sum of the unrounded p. The base of a row
 * is its running max, moved only when the max grows by more than 2^8 (p <= 256). */

/* The quantisation step alone. Inputs as in wan_attention_fwd (bf16, head_dim 128).
 * Outputs (device, caller-owned): q_codes [B, Lq, H*128] E4M3 bytes; q_scale
 * [B, Lq, H] fp32; k_codes [B, Lk, H*128]; vt_codes [B, H*128, vt_stride] (v
 * transposed: row = head dim, column = key; vt_stride % 64 == 0, vt_stride >= Lk;
 * columns from Lk to the next multiple of 64 are written as code 0); kv_scale [B, H, 2]
 * fp32 = (k scale, v scale), also used as scratch while the work runs. Five kernels. */
int wan_attention_fp8_quantize(const wan_dit_config* cfg, const void* q, int64_t q_row_stride, int q_col0,
                               const void* k, int64_t k_row_stride, int k_col0,
                               const void* v, int64_t v_row_stride, int v_col0,
                               int B, int heads, int Lq, int Lk, int head_dim,
                               void* q_codes, float* q_scale, void* k_codes, void* vt_codes, int64_t vt_stride,
                               float* kv_scale, void* stream);

/* softmax(q k^T / sqrt(d)) v on the E4M3 operands above: the same arguments and output
 * as wan_attention_fwd; the workspace (required, wan_attention_fp8_workspace_bytes)
 * holds the codes and scales, and the key-split scratch of a partial last wave. */
int wan_attention_fp8_fwd(const wan_dit_config* cfg, const void* q, int64_t q_row_stride, int q_col0,
                          const void* k, int64_t k_row_stride, int k_col0,
                          const void* v, int64_t v_row_stride, int v_col0,
                          void* o, int64_t o_row_stride, int o_col0,
                          int B, int heads, int Lq, int Lk, int head_dim, void* workspace, size_t ws_bytes,
                          void* stream);

/* Bytes of the wan_attention_fp8_fwd workspace for B samples, Lq queries, Lk keys. */
size_t wan_attention_fp8_workspace_bytes(const wan_dit_config* cfg, int B, int Lq, int Lk);

/* ---- tracing ------------------------------------------------------------------- */

/* Total number of kernels this library has launched in this process. */
int64_t wan_launch_count(void);

/* Turn per-launch CUDA-event timing on (1) or off (0). While on, each launch is
 * bracketed by events on its stream (a fixed pool of 16384 pairs per process). */
int wan_trace_enable(int on);

/* Drop all recorded launch timings. */
int wan_trace_reset(void);

/* Synchronise on the recorded events and return the total device time (ms) and the
 * number of timed launches of one wan_kernel_kind since the last reset. */
int wan_trace_read(int kind, double* total_ms, int64_t* launches);

/* Per-launch records since the last reset, in launch order (host arrays of `cap`
 * entries): kind, device time (ms) and algorithmic work - FLOPs (2 per multiply-add)
 * for GEMM and attention launches, bytes read + written for the others. Returns the
 * number of records written (<= cap) or a negative wan_status. */
int wan_trace_launches(int cap, int* kinds, double* ms, double* work);

#ifdef __cplusplus
}
#endif
#endif /* WAN_H */
