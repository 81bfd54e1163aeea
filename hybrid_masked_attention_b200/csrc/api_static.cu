// Allocation-free variant of the Target-layer backward.
//
// Some callers cannot allocate device memory at all: code that runs inside a
// memory pool owned by someone else, a framework whose allocator must not be
// re-entered from this call site, or a process that has reserved every byte it
// may touch up front.  mtfm_attn_target_bwd needs a caller-provided scratch
// block (dA as bf16 hi/lo parts and the per-block dgamma/dbeta partials);
// mtfm_attn_target_bwd_static instead uses a fixed scratch array that lives in
// the library image itself, so the caller passes only inputs and outputs.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library's device code holds kStaticScratchBytes for the life of the process.
// With CUDA's lazy module loading (the default), that device memory is committed
// when this file's module is first loaded on a device, which is the first call
// of this entry point there (its cudaGetSymbolAddress); a caller that reserves
// the rest of its device memory, or captures streams, afterwards should make one
// call first.  Later calls allocate nothing.  Host code cannot use the array's
// name as a device address, so every call looks the address up with
// cudaGetSymbolAddress on the device of the call's stream, which must be the
// current device (after a device reset the lookup simply finds the reloaded
// module).  All calls share the one array, so calls whose work overlaps on the
// GPU (different streams, or different host threads on one stream without
// ordering) race on it.  Nothing in it needs to start at zero: every byte the
// backward reads was written earlier in the same call.
#include "mtfm_internal.cuh"

namespace {

constexpr size_t kStaticScratchBytes = size_t(24) << 20;  // 24 MiB

__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch on the current device, which must also be the
// device of `stream` (NULL: the legacy stream of the current device).
mtfm_status static_scratch(void* stream, void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return MTFM_ERR_CUDA;
  if (stream) {
    int sdev = -1;
    if (cudaStreamGetDevice(static_cast<cudaStream_t>(stream), &sdev) != cudaSuccess) return MTFM_ERR_CUDA;
    if (sdev != dev) return MTFM_ERR_INVALID_ARG;
  }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return MTFM_ERR_CUDA;
  *out = p;
  return MTFM_OK;
}

}  // namespace

extern "C" mtfm_status mtfm_attn_target_bwd_static(
    const mtfm_cfg* cfg, const void* d_meta, const uint16_t* d_q, const uint16_t* d_k,
    const uint16_t* d_v, const uint16_t* d_u, const float* d_gamma, const float* d_beta,
    const float* d_a, const float* d_stats, const uint16_t* d_dy, float* d_dq, float* d_dk,
    float* d_dv, float* d_du, float* d_dgamma, float* d_dbeta, void* stream) {
  const size_t need = mtfm_bwd_workspace_bytes(cfg, 1);
  if (need == 0) return MTFM_ERR_INVALID_ARG;
  if (need > kStaticScratchBytes) return MTFM_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = nullptr;
  const mtfm_status s = static_scratch(stream, &scratch);
  if (s != MTFM_OK) return s;
  return mtfm_attn_target_bwd(cfg, d_meta, d_q, d_k, d_v, d_u, d_gamma, d_beta, d_a, d_stats, d_dy,
                              d_dq, d_dk, d_dv, d_du, d_dgamma, d_dbeta, scratch,
                              kStaticScratchBytes, stream);
}
