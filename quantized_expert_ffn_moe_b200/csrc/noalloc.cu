// moe_layer_forward_noalloc: the layer forward for callers that cannot
// allocate device memory.  Its scratch lives in a fixed array compiled into
// this library instead of a caller-provided workspace.
#include "moe_internal.cuh"

#include <cuda.h>

#include <mutex>

namespace {

// The scratch of the layer forward.  Every device that loads the library holds
// one copy of it until the process exits.
constexpr size_t kScratchBytes = MOE_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

// The array's name is a host-side handle, not a device address: the address
// comes from cudaGetSymbolAddress, looked up with the device current.  The
// module (and with it the array) is loaded per CUDA context, so the address is
// cached per device together with the id of the context it belongs to; when
// the context has been destroyed and re-created (cudaDeviceReset, or the
// primary context released and retained again) the id changes and the address
// is looked up again.
constexpr int kMaxDevices = 64;
struct Entry {
  unsigned long long ctx_id;
  void* addr;
};
std::mutex g_mu;
Entry g_entries[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <typename F>
F driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<F>(p);
}

// Id of the calling thread's current context, 0 when none is current.
bool current_ctx_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  if (!get_current || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS) return false;
  *id = 0;
  return !ctx || get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of g_scratch on the current device and context.
int scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  unsigned long long id = 0;
  const bool have = current_ctx_id(&id) && id != 0;     // false also for a destroyed context
  Entry& en = g_entries[dev];
  if (!have || en.addr == nullptr || en.ctx_id != id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
    if (!current_ctx_id(&id) || id == 0) return MOE_ERR_CUDA;    // the lookup made the context current
    en.addr = p;
    en.ctx_id = id;
  }
  *out = en.addr;
  return MOE_OK;
}

}  // namespace

extern "C" int moe_layer_forward_noalloc(const moe_config* cfg, const moe_layer_weights* w, const uint16_t* x,
                                         int32_t T, uint16_t* y, void* stream) {
  // the same checks, in the same order, as moe_layer_forward; then the size
  // limit of the fixed scratch in place of the workspace check
  int st = moe::check_layer_args(cfg, w, x, T, y);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if (moe_workspace_bytes(cfg, T) > kScratchBytes) return MOE_ERR_WORKSPACE;
  void* scratch = nullptr;
  if ((st = scratch_for_current_device(&scratch)) != MOE_OK) return st;
  return moe_layer_forward(cfg, w, x, T, y, scratch, kScratchBytes, stream);
}

extern "C" int moe_noalloc_device_status(int32_t* code_out) {
  if (!code_out) return MOE_ERR_INVALID_ARG;
  void* scratch = nullptr;
  const int st = scratch_for_current_device(&scratch);
  if (st != MOE_OK) return st;
  return moe_device_status(scratch, code_out);
}
