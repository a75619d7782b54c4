// Patchify for callers that cannot allocate device memory.
//
// wan_patchify needs a scratch buffer for the gathered 2x2 patches, which the caller
// passes as a workspace. Some callers cannot provide one: code that runs where the
// CUDA allocator must not be called (inside a host callback or an allocation-free
// real-time loop), plug-ins handed only input and output pointers by their host
// framework, or callers under a memory budget that forbids new device allocations
// after start-up. wan_patchify_noalloc serves them: its scratch is a fixed array in the
// library's own device memory, so the call needs nothing beyond its inputs and outputs.
//
// The array is g_patchify_scratch below: WAN_PATCHIFY_NOALLOC_SCRATCH_BYTES (16 MiB) in
// every device that loads the library, held until the process exits. Host code cannot
// use the array's name as a device address (on the host it is only a stand-in symbol),
// so the first call on each device looks the address up with cudaGetSymbolAddress,
// with that device current, and caches it; later calls reuse it. That first call should
// therefore come before any stream capture. The cached address is tagged with the CUDA
// context it came from: after a device reset (a new primary context, which reloads the
// module, possibly at another address) the next call looks it up again, so that call
// too should come before any capture. Every call shares the one array, so calls whose
// work overlaps on the GPU (different streams, or different host threads on one device)
// race on it and must be serialised by the caller. Nothing in the array has to start at
// zero: each call writes every scratch byte it later reads.
#include <cuda_runtime.h>

#include "internal.h"

namespace wan {
namespace {

static __device__ __align__(256) unsigned char g_patchify_scratch[WAN_PATCHIFY_NOALLOC_SCRATCH_BYTES];

// Device address of g_patchify_scratch on the current device.
int patchify_scratch(void** out) {
  static SymbolCache cache;
  return cache.get(&g_patchify_scratch, out);
}

}  // namespace
}  // namespace wan

using namespace wan;

extern "C" int wan_patchify_noalloc(const wan_dit_config* cfg, const void* latent, int B, int F, int H, int W,
                                    const void* w_p, const void* b_p, float* x_out, void* stream) {
  // The same argument checks, in the same order, as wan_patchify.
  int st = check_cfg(cfg);
  if (st == WAN_OK) st = check_ptr(latent);
  if (st == WAN_OK) st = check_ptr(w_p);
  if (st == WAN_OK) st = check_opt_ptr(b_p);
  if (st == WAN_OK) st = check_ptr(x_out);
  if (st != WAN_OK) return st;
  if (B < 0 || F < 0 || H < 0 || W < 0 || H % 2 != 0 || W % 2 != 0) return WAN_ERR_SHAPE;
  const size_t rows = static_cast<size_t>(B) * F * (H / 2) * (W / 2);
  if (rows >= (size_t(1) << 31)) return WAN_ERR_SHAPE;
  const int K = cfg->in_ch * 4;
  if (rows * K * dtype_size(cfg->dtype) > WAN_PATCHIFY_NOALLOC_SCRATCH_BYTES) return WAN_ERR_SHAPE;
  void* scratch = nullptr;
  st = patchify_scratch(&scratch);
  if (st != WAN_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int M = static_cast<int>(rows);
  st = launch_patch_gather(latent, B, cfg->in_ch, F, H, W, scratch, cfg->dtype, s);
  if (st != WAN_OK) return st;
  GemmEpi ep{};
  ep.kind = WAN_EPI_F32;
  ep.ldo = cfg->dim;
  ep.rows_per_batch = 1;
  if (cfg->dtype == WAN_BF16) return launch_gemm_tc(scratch, K, w_p, b_p, x_out, M, cfg->dim, K, 0, ep, s);
  return launch_gemm_simt(static_cast<const float*>(scratch), K, static_cast<const float*>(w_p),
                          static_cast<const float*>(b_p), x_out, M, cfg->dim, K, 0, ep, s);
}
