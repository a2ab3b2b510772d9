// lowram_decode_step_static: the decode step with its scratch in a fixed device array of
// this library instead of a caller-provided workspace.
//
// Who needs it: callers that cannot allocate device memory at the point where they
// decode. Examples are a serving loop whose memory pool is fully reserved, a runtime that
// forbids allocation after start-up, and a plugin that owns no allocator. The entry point
// itself allocates nothing. It needs only the context (created earlier) and the caller's
// input and output buffers.
//
// The scratch is a file-scope array of kStaticScratchBytes (32 MiB). Every GPU that loads
// the library holds it until the process exits. It is as large as the decode workspace of
// a 128K-token, batch-8 Llama-3-8B-shaped layer.
#include <cuda_runtime.h>

#include <mutex>

#include "lowram_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

// Device-side scratch. In host code this name is only a stand-in: its device address
// comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch on `device` (looked up on first use, with that device
// current), or nullptr when the runtime refuses.
void* scratch_on(int device) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (device < 0 || device >= kMaxDevices) return nullptr;
  if (g_scratch_addr[device]) return g_scratch_addr[device];
  int prev = -1;
  if (cudaGetDevice(&prev) != cudaSuccess) return nullptr;
  if (prev != device && cudaSetDevice(device) != cudaSuccess) return nullptr;
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
  if (prev != device) cudaSetDevice(prev);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  g_scratch_addr[device] = p;
  return p;
}

}  // namespace

extern "C" lowram_status lowram_decode_step_static(lowram_ctx* ctx, const lowram_cache* cache,
                                                   const lowram_layer_params* params,
                                                   const void* q, void* out, int32_t* sel_out,
                                                   void* stream) {
  if (!ctx) return LOWRAM_ERR_INVALID_ARG;
  size_t need = 0;
  const lowram_status st =
      lowram_workspace_size(lowram::ctx_config(ctx), LOWRAM_OP_DECODE, &need);
  if (st != LOWRAM_OK) return st;
  if (need > kStaticScratchBytes) return LOWRAM_ERR_WORKSPACE;
  void* scratch = scratch_on(lowram::ctx_device(ctx));
  if (!scratch) return LOWRAM_ERR_CUDA;
  return lowram_decode_step(ctx, cache, params, q, out, sel_out, scratch, kStaticScratchBytes,
                            stream);
}
