// C ABI of libmoe.so: argument validation and launch sequencing.  The
// operation and the conventions are documented in include/moe_capi.h.
#include "moe_internal.cuh"


namespace moe {
cudaError_t launch_route_full(const moe_config& c, const uint16_t* router_w, const float* bias,
                              const uint16_t* x, int T, char* ws, const Layout& L, int* api_counts,
                              int* api_offsets, int* api_pairs, cudaStream_t s, int ep_rank, int ep_size);
}

using namespace moe;

namespace {

// Batches of up to this many tokens take the decode path (grouped GEMV on CUDA
// cores); larger batches the tensor-core prefill path.
constexpr int kDecodeMaxTokens = 64;
// Single-layer batches from this size up may hand over to the tensor cores.
constexpr int kHybridMinTokens = 32;

int num_sms_current() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int validate_config(const moe_config* c) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (c->num_experts <= 0 || c->hidden <= 0 || c->inter <= 0 || c->top_k <= 0 || c->shared_inter < 0)
    return MOE_ERR_INVALID_ARG;
  if (c->num_experts > 1024 || c->num_experts % 32 != 0) return MOE_ERR_UNSUPPORTED;
  if (c->top_k > 16 || c->top_k > c->num_experts) return MOE_ERR_UNSUPPORTED;
  if (!((c->bits == 4 && (c->block == 32 || c->block == 128)) || (c->bits == 2 && c->block == 16)))
    return MOE_ERR_UNSUPPORTED;
  if (c->half_levels != 0 && c->half_levels != 1) return MOE_ERR_UNSUPPORTED;
  if (c->scale_fmt != 0 && c->scale_fmt != 1) return MOE_ERR_UNSUPPORTED;
  if (c->scale_fmt == 1 && (c->block == 128 || c->half_levels)) return MOE_ERR_UNSUPPORTED;
  const int H = c->hidden;
  if (!(H == 256 || H == 512 || H == 1024 || H == 2048 || H == 4096)) return MOE_ERR_UNSUPPORTED;
  if (c->inter % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (c->shared_inter != 0 && c->shared_inter != c->inter) return MOE_ERR_UNSUPPORTED;
  if (!decode_shape_supported(c->bits, H, c->inter)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

int validate_weights(const moe_config* c, const moe_layer_weights* w) {
  if (!w) return MOE_ERR_INVALID_ARG;
  const void* req[] = {w->gate_up_codes, w->gate_up_scales, w->down_codes, w->down_scales, w->router_w};
  for (const void* p : req)
    if (!p || !aligned(p, 16)) return MOE_ERR_INVALID_ARG;
  if (c->shared_inter > 0) {
    const void* sh[] = {w->shared_gate_up_codes, w->shared_gate_up_scales, w->shared_down_codes,
                        w->shared_down_scales};
    for (const void* p : sh)
      if (!p || !aligned(p, 16)) return MOE_ERR_INVALID_ARG;
  }
  if (w->router_bias && !aligned(w->router_bias, 4)) return MOE_ERR_INVALID_ARG;
  if (w->shared_gate_w && (c->shared_inter == 0 || !aligned(w->shared_gate_w, 16))) return MOE_ERR_INVALID_ARG;
  // fp8 block scales come with one fp32 scale per row; fp16 scales with none
  const void* rs[] = {w->gate_up_row_scales, w->down_row_scales};
  const void* srs[] = {w->shared_gate_up_row_scales, w->shared_down_row_scales};
  for (const void* p : rs)
    if (c->scale_fmt == 1 ? (!p || !aligned(p, 16)) : p != nullptr) return MOE_ERR_INVALID_ARG;
  for (const void* p : srs)
    if (c->scale_fmt == 1 && c->shared_inter > 0 ? (!p || !aligned(p, 16)) : (c->scale_fmt == 0 && p != nullptr))
      return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

int check_ws(const moe_config* c, int T, void* ws, size_t ws_bytes) {
  if (!ws || !aligned(ws, 256)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < moe_workspace_bytes(c, T)) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

thread_local int g_last_cuda_error = 0;

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return MOE_OK;
  g_last_cuda_error = int(e);
  return MOE_ERR_CUDA;
}

// Optional per-phase event recording (moe_profile_begin / moe_profile_end).
struct Profile {
  bool on = false;
  int cap = 0, used = 0;
  cudaEvent_t* ev = nullptr;    // [cap][5]
  unsigned char* fused = nullptr;  // [cap] call ran as one fused kernel
};
Profile g_prof;

void prof_mark(int call, int phase, cudaStream_t s) {
  if (call >= 0) cudaEventRecord(g_prof.ev[call * 5 + phase], s);
}

// One layer on the stream: route, gate/up + SwiGLU, down, combine.
int run_layer(const LayerArgs& a) {
  const int call = (g_prof.on && g_prof.used < g_prof.cap) ? g_prof.used++ : -1;
  prof_mark(call, 0, a.stream);
  cudaError_t e = launch_route_full(a.cfg, a.w.router_w, a.w.router_bias, a.x, a.T, a.ws, a.L, nullptr,
                                    nullptr, nullptr, a.stream, a.ep_rank, a.ep_size);
  if (e != cudaSuccess) return cuda_status(e);
  prof_mark(call, 1, a.stream);
  LayerArgs comb = a;
  if (a.T > kDecodeMaxTokens && prefill_supported(a.cfg)) {
    e = launch_prefill_ffn(a);
    if (call >= 0) cudaEventRecord(g_prof.ev[call * 5 + 2], a.stream);
    comb.y_half = 1;                      // the tensor-core down pass writes fp16 rows
  } else {
    e = launch_decode_ffn(a, call >= 0 ? g_prof.ev[call * 5 + 2] : nullptr);
  }
  if (e != cudaSuccess) return cuda_status(e);
  prof_mark(call, 3, a.stream);
  e = launch_combine(comb);
  prof_mark(call, 4, a.stream);
  return cuda_status(e);
}

}  // namespace

namespace moe {
// Everything moe_layer_forward checks before it looks at the workspace, in the
// same order: the config, T, the weights, x and y (non-null, 16-byte aligned,
// not overlapping).  T == 0 passes (the call is then a no-op).
int check_layer_args(const moe_config* cfg, const moe_layer_weights* w, const uint16_t* x, int32_t T,
                     const uint16_t* y) {
  int st = validate_config(cfg);
  if (st != MOE_OK) return st;
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if ((st = validate_weights(cfg, w)) != MOE_OK) return st;
  if (!x || !y || !aligned(x, 16) || !aligned(y, 16)) return MOE_ERR_INVALID_ARG;
  const size_t bytes = size_t(T) * cfg->hidden * 2;
  const char* xb = reinterpret_cast<const char*>(x);
  const char* yb = reinterpret_cast<const char*>(y);
  if (xb < yb + bytes && yb < xb + bytes) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}
}  // namespace moe

extern "C" {

size_t moe_workspace_bytes(const moe_config* cfg, int32_t max_tokens) {
  if (validate_config(cfg) != MOE_OK || max_tokens < 0) return 0;
  return make_layout(*cfg, max_tokens).total;
}

int moe_route(const moe_config* cfg, const uint16_t* router_w, const float* router_bias, const uint16_t* x,
              int32_t T, int32_t* topk_idx, float* topk_w, int32_t* expert_counts, int32_t* expert_offsets,
              int32_t* pairs, void* workspace, size_t ws_bytes, void* stream) {
  int st = validate_config(cfg);
  if (st != MOE_OK) return st;
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!router_w || !aligned(router_w, 16) || !x || !aligned(x, 16) || !topk_idx || !topk_w)
    return MOE_ERR_INVALID_ARG;
  if (router_bias && !aligned(router_bias, 4)) return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(cfg, T, workspace, ws_bytes)) != MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  const Layout L = make_layout(*cfg, T);
  if (cudaMemsetAsync(ws + L.status, 0, ST_COUNT * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
  cudaError_t e = launch_route_full(*cfg, router_w, router_bias, x, T, ws, L, expert_counts, expert_offsets,
                                    pairs, s, 0, 1);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  const size_t n = size_t(T) * cfg->top_k;
  if (cudaMemcpyAsync(topk_idx, ws + L.topk_idx, n * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaMemcpyAsync(topk_w, ws + L.topk_w, n * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

int moe_layer_forward(const moe_config* cfg, const moe_layer_weights* w, const uint16_t* x, int32_t T,
                      uint16_t* y, void* workspace, size_t ws_bytes, void* stream) {
  int st = moe::check_layer_args(cfg, w, x, T, y);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if ((st = check_ws(cfg, T, workspace, ws_bytes)) != MOE_OK) return st;
  LayerArgs a{};
  a.cfg = *cfg; a.w = *w; a.T = T; a.x = x; a.y = y; a.residual = false; a.xhat_next = nullptr;
  a.ws = static_cast<char*>(workspace);
  a.L = make_layout(*cfg, T);
  a.num_sms = num_sms_current();
  a.stream = static_cast<cudaStream_t>(stream);
  int* status = reinterpret_cast<int*>(a.ws + a.L.status);
  if (T <= kDecodeMaxTokens && fused_supported(*cfg, T) && !w->shared_gate_w) {
    if (launch_status_reset(status, a.stream) != cudaSuccess) return MOE_ERR_CUDA;
    const int call = (g_prof.on && g_prof.used < g_prof.cap) ? g_prof.used++ : -1;
    prof_mark(call, 0, a.stream);
    // 32..64 tokens: the fused kernel routes and then either finishes the
    // layer or, when its cost model favours them, leaves it to the grouped
    // tensor-core kernels queued behind it (they do nothing otherwise)
    const int mode = decode_path_mode();
    const int hybrid = (T >= kHybridMinTokens && prefill_supported(*cfg) && mode != 1) ? (mode == 2 ? 2 : 1) : 0;
    cudaError_t e = launch_fused_decode(*cfg, w, 1, x, y, false, T, nullptr, a.ws, a.L, a.num_sms, a.stream, hybrid);
    if (e == cudaSuccess && hybrid) {
      a.gated = 1;
      a.y_half = 1;
      e = launch_prefill_ffn(a);
      if (e == cudaSuccess) e = launch_combine(a);
    }
    if (e == cudaSuccess) {
      for (int ph = 1; ph <= 4; ++ph) prof_mark(call, ph, a.stream);
      if (call >= 0) g_prof.fused[call] = 1;
      return MOE_OK;
    }
    if (e != cudaErrorCooperativeLaunchTooLarge) return cuda_status(e);
    (void)cudaGetLastError();        // cannot co-schedule one CTA per SM here: separate kernels
    if (call >= 0) g_prof.used--;
    return run_layer(a);              // the status words are already cleared
  }
  if (cudaMemsetAsync(status, 0, ST_COUNT * 4, a.stream) != cudaSuccess) return MOE_ERR_CUDA;
  return run_layer(a);
}

int moe_layer_forward_ep(const moe_config* cfg, const moe_layer_weights* w, const uint16_t* x, int32_t T,
                         int32_t ep_rank, int32_t ep_size, float* y_partial, void* workspace, size_t ws_bytes,
                         void* stream) {
  int st = validate_config(cfg);
  if (st != MOE_OK) return st;
  if (T < 0 || ep_size < 1 || ep_size > cfg->num_experts || ep_rank < 0 || ep_rank >= ep_size)
    return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!w) return MOE_ERR_INVALID_ARG;
  moe_config c = *cfg;
  moe_layer_weights wl = *w;
  if (ep_rank != 0) {                            // the shared expert (and its gate) belong to rank 0
    c.shared_inter = 0;
    wl.shared_gate_w = nullptr;
  }
  if ((st = validate_weights(&c, &wl)) != MOE_OK) return st;
  if (!x || !y_partial || !aligned(x, 16) || !aligned(y_partial, 16)) return MOE_ERR_INVALID_ARG;
  const char* xb = reinterpret_cast<const char*>(x);
  const char* yb = reinterpret_cast<const char*>(y_partial);
  if (xb < yb + size_t(T) * cfg->hidden * 4 && yb < xb + size_t(T) * cfg->hidden * 2) return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(cfg, T, workspace, ws_bytes)) != MOE_OK) return st;
  LayerArgs a{};
  a.cfg = c; a.w = wl; a.T = T; a.x = x; a.y = nullptr; a.residual = false; a.xhat_next = nullptr;
  a.ws = static_cast<char*>(workspace);
  a.L = make_layout(*cfg, T);
  a.num_sms = num_sms_current();
  a.stream = static_cast<cudaStream_t>(stream);
  a.ep_rank = ep_rank;
  a.ep_size = ep_size;
  a.y_f32 = y_partial;
  if (cudaMemsetAsync(a.ws + a.L.status, 0, ST_COUNT * 4, a.stream) != cudaSuccess) return MOE_ERR_CUDA;
  return run_layer(a);
}

int moe_stack_forward(const moe_config* cfg, const moe_layer_weights* layers, int32_t L, uint16_t* x_inout,
                      int32_t T, int32_t* topk_trace, void* workspace, size_t ws_bytes, void* stream) {
  int st = validate_config(cfg);
  if (st != MOE_OK) return st;
  if (T < 0 || L < 0 || !layers) return MOE_ERR_INVALID_ARG;
  if (T == 0 || L == 0) return MOE_OK;
  for (int l = 0; l < L; ++l)
    if ((st = validate_weights(cfg, &layers[l])) != MOE_OK) return st;
  if (!x_inout || !aligned(x_inout, 16)) return MOE_ERR_INVALID_ARG;
  if (topk_trace && !aligned(topk_trace, 4)) return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(cfg, T, workspace, ws_bytes)) != MOE_OK) return st;
  LayerArgs a{};
  a.cfg = *cfg; a.T = T;
  a.ws = static_cast<char*>(workspace);
  a.L = make_layout(*cfg, T);
  a.num_sms = num_sms_current();
  a.stream = static_cast<cudaStream_t>(stream);
  uint16_t* xhat = reinterpret_cast<uint16_t*>(a.ws + a.L.xhat);
  int* status = reinterpret_cast<int*>(a.ws + a.L.status);
  bool gated = false;
  for (int l = 0; l < L; ++l) gated = gated || layers[l].shared_gate_w != nullptr;
  const bool fused = T <= kDecodeMaxTokens && fused_supported(*cfg, T) && !gated;
  if (fused) {
    if (launch_status_reset(status, a.stream) != cudaSuccess) return MOE_ERR_CUDA;
  } else if (cudaMemsetAsync(status, 0, ST_COUNT * 4, a.stream) != cudaSuccess) {
    return MOE_ERR_CUDA;
  }
  if (fused) {
    const cudaError_t e = launch_fused_decode(*cfg, layers, L, x_inout, x_inout, true, T, topk_trace, a.ws, a.L,
                                              a.num_sms, a.stream);
    if (e == cudaSuccess) return MOE_OK;
    if (e != cudaErrorCooperativeLaunchTooLarge) return cuda_status(e);
    (void)cudaGetLastError();
  }
  if (launch_rmsnorm(x_inout, xhat, T, cfg->hidden, a.stream) != cudaSuccess) return MOE_ERR_CUDA;
  for (int l = 0; l < L; ++l) {
    a.w = layers[l];
    a.x = xhat;
    a.y = x_inout;
    a.residual = true;
    a.xhat_next = (l + 1 < L) ? xhat : nullptr;
    if ((st = run_layer(a)) != MOE_OK) return st;
    if (topk_trace) {
      const size_t n = size_t(T) * cfg->top_k;
      if (cudaMemcpyAsync(topk_trace + size_t(l) * n, a.ws + a.L.topk_idx, n * 4, cudaMemcpyDeviceToDevice,
                          a.stream) != cudaSuccess)
        return MOE_ERR_CUDA;
    }
  }
  return MOE_OK;
}

int moe_device_status(const void* workspace, int32_t* code_out) {
  if (!workspace || !code_out) return MOE_ERR_INVALID_ARG;
  int32_t v[2] = {0, 0};
  if (cudaMemcpy(v, workspace, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  *code_out = v[0];
  return v[0] == 0 ? MOE_OK : MOE_ERR_DEVICE_CHECK;
}

int moe_dequant_rows_scaled(const moe_config* cfg, const uint8_t* codes, const void* scales,
                            const float* row_scales, int32_t row0, int32_t rows, int32_t cols, float* out,
                            void* stream) {
  if (!cfg || !codes || !scales || !out || row0 < 0 || rows < 0 || cols <= 0) return MOE_ERR_INVALID_ARG;
  if (!((cfg->bits == 4 && (cfg->block == 32 || cfg->block == 128)) || (cfg->bits == 2 && cfg->block == 16)))
    return MOE_ERR_UNSUPPORTED;
  if (cfg->half_levels != 0 && cfg->half_levels != 1) return MOE_ERR_UNSUPPORTED;
  if (cfg->scale_fmt != 0 && cfg->scale_fmt != 1) return MOE_ERR_UNSUPPORTED;
  if ((cfg->scale_fmt == 1) != (row_scales != nullptr)) return MOE_ERR_INVALID_ARG;
  if (cols % cfg->block != 0 || (cols * cfg->bits / 8) % 4 != 0) return MOE_ERR_UNSUPPORTED;
  if (!aligned(codes, 4) || !aligned(scales, cfg->scale_fmt ? 1 : 2) || !aligned(out, 4) ||
      (row_scales && !aligned(row_scales, 4)))
    return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  return cuda_status(launch_dequant_rows(cfg->bits, cfg->block, cfg->half_levels, cfg->scale_fmt, codes, scales,
                                         row_scales, row0, rows, cols, out, static_cast<cudaStream_t>(stream)));
}

int moe_dequant_rows(const moe_config* cfg, const uint8_t* codes, const uint16_t* scales, int32_t row0,
                     int32_t rows, int32_t cols, float* out, void* stream) {
  if (cfg && cfg->scale_fmt != 0) return MOE_ERR_UNSUPPORTED;
  return moe_dequant_rows_scaled(cfg, codes, scales, nullptr, row0, rows, cols, out, stream);
}

int moe_profile_begin(int32_t max_calls) {
  if (max_calls <= 0 || g_prof.on) return MOE_ERR_INVALID_ARG;
  g_prof.ev = new cudaEvent_t[size_t(max_calls) * 5];
  g_prof.fused = new unsigned char[max_calls]();
  for (int i = 0; i < max_calls * 5; ++i)
    if (cudaEventCreate(&g_prof.ev[i]) != cudaSuccess) return MOE_ERR_CUDA;
  g_prof.cap = max_calls;
  g_prof.used = 0;
  g_prof.on = true;
  return MOE_OK;
}

int moe_profile_end(float* ms_out, int32_t* calls) {
  if (!g_prof.on || !ms_out || !calls) return MOE_ERR_INVALID_ARG;
  int st = MOE_OK;
  for (int p = 0; p < 5; ++p) ms_out[p] = 0.f;
  for (int c = 0; c < g_prof.used; ++c) {
    for (int p = 0; p < 4; ++p) {
      float ms = 0.f;
      if (cudaEventSynchronize(g_prof.ev[c * 5 + p + 1]) != cudaSuccess ||
          cudaEventElapsedTime(&ms, g_prof.ev[c * 5 + p], g_prof.ev[c * 5 + p + 1]) != cudaSuccess)
        st = MOE_ERR_CUDA;
      ms_out[g_prof.fused[c] ? 4 : p] += ms;
    }
  }
  *calls = g_prof.used;
  for (int i = 0; i < g_prof.cap * 5; ++i) cudaEventDestroy(g_prof.ev[i]);
  delete[] g_prof.ev;
  delete[] g_prof.fused;
  g_prof = Profile{};
  return st;
}

int moe_last_cuda_error(void) { return g_last_cuda_error; }

void moe_debug_fused_timing(unsigned long long* device_buf) { set_fused_timing(device_buf); }

void moe_debug_prefill_timing(unsigned long long* device_buf) { set_prefill_timing(device_buf); }

void moe_debug_decode_path(int32_t mode) { set_decode_path_mode(mode >= 0 && mode <= 2 ? mode : 0); }

const char* moe_status_str(int status) {
  switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument (null, misaligned or negative)";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape or format";
    case MOE_ERR_WORKSPACE: return "workspace smaller than moe_workspace_bytes()";
    case MOE_ERR_CUDA: return "a CUDA runtime call failed";
    case MOE_ERR_DEVICE_CHECK: return "a device-side check failed";
    case MOE_ERR_TIMEOUT: return "a bounded device wait timed out";
    default: return "unknown status";
  }
}

}  // extern "C"
