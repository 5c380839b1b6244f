// moe_layer_forward_noalloc: the layer forward for callers that cannot
// allocate device memory.  Its scratch lives in a fixed array compiled into
// this library instead of a caller-provided workspace.
#include "moe_internal.cuh"

#include <mutex>

namespace {

// The scratch of the layer forward.  Every device that loads the library holds
// one copy of it until the process exits.
constexpr size_t kScratchBytes = MOE_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of g_scratch on the current device, looked up once per
// device (the symbol's name is only a host-side handle).
int scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" int moe_layer_forward_noalloc(const moe_config* cfg, const moe_layer_weights* w, const uint16_t* x,
                                         int32_t T, uint16_t* y, void* stream) {
  const size_t need = moe_workspace_bytes(cfg, T);
  if (need == 0) return cfg ? (T < 0 ? MOE_ERR_INVALID_ARG : MOE_ERR_UNSUPPORTED) : MOE_ERR_INVALID_ARG;
  if (need > kScratchBytes) return MOE_ERR_WORKSPACE;
  void* scratch = nullptr;
  const int st = scratch_for_current_device(&scratch);
  if (st != MOE_OK) return st;
  return moe_layer_forward(cfg, w, x, T, y, scratch, kScratchBytes, stream);
}
