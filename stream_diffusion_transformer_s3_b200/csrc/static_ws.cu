// zdit_block_forward_static: the block forward for callers that cannot allocate.
//
// Some callers of this library cannot call cudaMalloc at all: a plugin inside a host
// framework that has already reserved (nearly) all device memory for its own pool, so
// a fresh allocation fails, or a latency-critical loop where cudaMalloc's implicit
// device-wide synchronization is not acceptable.  zdit_block_forward needs a caller
// workspace; this entry point instead uses one scratch array that the library owns as
// a file-scope device variable, so a call allocates nothing.
//
// Cost: every GPU that loads this library holds kStaticScratchBytes (40 MiB) until
// the process exits.  Calls whose workspace would exceed that are rejected.
#include <cuda_runtime.h>

#include "../../include/zdit.h"
#include "internal.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(40) << 20;  // 40 MiB

// The shared scratch.  In host code this name is only a host-side handle of the
// device variable, never a device address: the address is looked up on the current
// device with cudaGetSymbolAddress and passed to the kernels.
static __device__ __align__(256) unsigned char g_block_scratch[kStaticScratchBytes];

// Device address of g_block_scratch on the current device, or nullptr if the lookup
// fails.  Looked up on every call rather than cached: after cudaDeviceReset (or a
// primary-context release and re-creation) the module is loaded again and the array
// may sit at another address.  Once the module is loaded the lookup is cheap; the
// first one on a device loads the module.
void* scratch_on_current_device() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_block_scratch) != cudaSuccess) return nullptr;
  return p;
}

}  // namespace

extern "C" ZDIT_API zdit_status zdit_block_forward_static(const zdit_block_cfg* cfg, const zdit_block_weights* w,
                                                          const zdit_varlen* varlen, float* x, const float* temb,
                                                          const float* rope_cos, const float* rope_sin,
                                                          void* stream) {
  // the same checks, in the same order, as zdit_block_forward (minus the workspace)
  const zdit_status v = zdit::check_block_call(cfg, w, varlen, x, temb, rope_cos, rope_sin, nullptr, false);
  if (v != ZDIT_OK) return v;
  const int64_t T = varlen->cu_seqlens_host[varlen->batch];
  const size_t need = zdit_block_workspace_bytes(cfg, T, varlen->batch);
  if (need == 0) return ZDIT_ERR_SHAPE;
  if (need > kStaticScratchBytes) return ZDIT_ERR_WORKSPACE;  // too many tokens for the static scratch
  void* scratch = scratch_on_current_device();
  if (scratch == nullptr) return ZDIT_ERR_CUDA;
  // Every workspace region is written before it is read within a call, except the
  // per-band arrival counters of the out and down projections: those are zeroed by the
  // block's launch sequence at the start of each call (its band state lives for one call
  // only), so the previous call's contents never leak into this one.
  return zdit_block_forward(cfg, w, varlen, x, temb, rope_cos, rope_sin, scratch, kStaticScratchBytes, stream);
}
