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
// the library holds it until the process exits (or until the device's context is
// destroyed, e.g. by cudaDeviceReset). It is as large as the decode workspace of a
// 128K-token, batch-8 Llama-3-8B-shaped layer.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "lowram_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

// Device-side scratch. In host code this name is only a stand-in: its device address
// comes from cudaGetSymbolAddress, with the device current.
static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

// The address is cached per device together with the unique id of the CUDA context it
// was looked up in. A device reset destroys that context and the module with it; the
// array can then sit at a new address in the next context, whose id differs, so the next
// call looks the address up again instead of using a stale one.
struct ScratchEntry {
  unsigned long long ctx_id;
  void* addr;
};
std::mutex g_mu;
ScratchEntry g_scratch[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

template <typename Fn>
Fn driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(p);
}

// Unique id of the calling thread's current context (0 when it cannot be read).
unsigned long long current_ctx_id() {
  static CtxGetCurrentFn get_cur = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  CUcontext c = nullptr;
  unsigned long long id = 0;
  if (!get_cur || !get_id || get_cur(&c) != CUDA_SUCCESS || !c ||
      get_id(c, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of the scratch on `device` in its current context, looked up with that
// device current on the first call in each context; nullptr when the runtime refuses.
void* scratch_on(int device) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (device < 0 || device >= kMaxDevices) return nullptr;
  int prev = -1;
  if (cudaGetDevice(&prev) != cudaSuccess) return nullptr;
  // since CUDA 12, cudaSetDevice also makes the device's primary context current
  if (cudaSetDevice(device) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  void* p = nullptr;
  cudaError_t e = cudaSuccess;
  const unsigned long long id = current_ctx_id();
  ScratchEntry& ent = g_scratch[device];
  if (id != 0 && ent.ctx_id == id && ent.addr) {
    p = ent.addr;
  } else {
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e == cudaSuccess) {
      ent.ctx_id = current_ctx_id();   // 0 (unreadable) never matches: looked up again
      ent.addr = p;
    }
  }
  if (prev != device) cudaSetDevice(prev);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
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
