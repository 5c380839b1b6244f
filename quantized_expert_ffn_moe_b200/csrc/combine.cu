// Gate-weighted combine: out[t] = g_t Y[shared, t] + sum_j Y[(t, j)] in fixed
// slot order (the gate weight is already inside Y), fp32, rounded once to
// bf16; g_t = 1, or sigmoid(x_t . w) when the layer has a shared-expert gate.
// Y rows are fp32 (decode GEMV) or fp16 (tensor-core path, y_half).
// The shared expert is added with weight 1 ("How a 125B Model Reaches 100
// Tok/s on an RTX 4090", section "The model is large on paper, sparse in
// practice": 10 routed experts plus one shared expert are active per token).
// In the stack the residual add and the next layer's RMSNorm are fused here:
// x <- bf16(x + out), xhat <- bf16(x / sqrt(mean(x^2) + 1e-6)).
// Expert-parallel share: pairs whose expert another rank owns carry position
// -1 and are skipped, and the partial sum is written in fp32 (out_f32) for
// the all-reduce over ranks.
#include "moe_internal.cuh"

namespace moe {

namespace {

constexpr int kCombThreads = 256;

// YH: the Y rows are fp16 (each kernel instance holds one row format only,
// so the fp16 one keeps its registers low enough for six CTAs per SM).
template <bool YH>
__global__ void __launch_bounds__(kCombThreads) combine_kernel(
    const float* __restrict__ Y, const int* __restrict__ inv, int T, int k, int H, int shared,
    uint16_t* __restrict__ out, int residual, uint16_t* __restrict__ xhat_next, float* __restrict__ out_f32,
    const int* __restrict__ gate, const uint16_t* __restrict__ xin, const uint16_t* __restrict__ sgate_w) {
  constexpr bool y_half = YH;
  pdl_wait();
  if (gate && __ldcg(gate) == 0) {                // the fused decode kernel kept (and combined) the layer
    pdl_launch_dependents();
    return;
  }
  const int t = blockIdx.x;
  const int P_routed = T * k;
  __shared__ int pos[16];
  __shared__ float gred[kCombThreads / 32];
  if (threadIdx.x < k) pos[threadIdx.x] = inv[t * k + threadIdx.x];
  // the shared expert's weight: 1, or sigmoid(x . w) with the layer input x
  // (exact bf16 products, fp32 sum)
  float gsh = 1.f;
  if (shared && sgate_w) {
    float a = 0.f;
    for (int h0 = threadIdx.x * 8; h0 < H; h0 += kCombThreads * 8) {
      const uint4 xv = *reinterpret_cast<const uint4*>(xin + size_t(t) * H + h0);
      const uint4 wv = *reinterpret_cast<const uint4*>(sgate_w + h0);
      const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w}, ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a = fmaf(__uint_as_float(xw[i] << 16), __uint_as_float(ww[i] << 16), a);
        a = fmaf(__uint_as_float(xw[i] & 0xFFFF0000u), __uint_as_float(ww[i] & 0xFFFF0000u), a);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
    if ((threadIdx.x & 31) == 0) gred[threadIdx.x >> 5] = a;
    __syncthreads();
    float z = 0.f;
    for (int i = 0; i < kCombThreads / 32; ++i) z += gred[i];
    gsh = 1.f / (1.f + expf(-z));
  }
  __syncthreads();
  float ss = 0.f;
  constexpr int VPT = 8;                      // elements per thread per step
  for (int h0 = threadIdx.x * VPT; h0 < H; h0 += kCombThreads * VPT) {
    // 8 consecutive Y values of row p, in fp32
    auto yrow = [&](int p, float (&o)[VPT]) {
      if (y_half) {
        const uint4 hv = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(Y) + size_t(p) * H + h0);
        const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __half22float2(u32_as_h2(hw[i]));
          o[2 * i] = f.x;
          o[2 * i + 1] = f.y;
        }
      } else {
        const float4 a = *reinterpret_cast<const float4*>(Y + size_t(p) * H + h0);
        const float4 b = *reinterpret_cast<const float4*>(Y + size_t(p) * H + h0 + 4);
        o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w; o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
      }
    };
    float acc[VPT];
    if (shared) {
      float yv[VPT];
      yrow(P_routed + t, yv);
#pragma unroll
      for (int i = 0; i < VPT; ++i) acc[i] = gsh * yv[i];
    } else {
#pragma unroll
      for (int i = 0; i < VPT; ++i) acc[i] = 0.f;
    }
    if (YH) {
      // fp16 rows: four rows' loads in flight before their adds (slot order kept)
      for (int j0 = 0; j0 < k; j0 += 4) {
        uint4 hv[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (j0 + j < k && pos[j0 + j] >= 0)
            hv[j] = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(Y) + size_t(pos[j0 + j]) * H + h0);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (j0 + j < k && pos[j0 + j] >= 0) {
            const uint32_t hw[4] = {hv[j].x, hv[j].y, hv[j].z, hv[j].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 f = __half22float2(u32_as_h2(hw[i]));
              acc[2 * i] += f.x;
              acc[2 * i + 1] += f.y;
            }
          }
        }
      }
    } else {
      for (int j = 0; j < k; ++j) {
        if (pos[j] < 0) continue;                 // expert owned by another rank
        float yv[VPT];
        yrow(pos[j], yv);
#pragma unroll
        for (int i = 0; i < VPT; ++i) acc[i] += yv[i];
      }
    }
    if (out_f32) {
      float* fd = out_f32 + size_t(t) * H + h0;
      *reinterpret_cast<float4*>(fd) = make_float4(acc[0], acc[1], acc[2], acc[3]);
      *reinterpret_cast<float4*>(fd + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
      continue;
    }
    uint16_t* dst = out + size_t(t) * H + h0;
    if (residual) {
      const uint4 xv = *reinterpret_cast<const uint4*>(dst);
      const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] += __uint_as_float(xw[i] << 16);
        acc[2 * i + 1] += __uint_as_float(xw[i] & 0xFFFF0000u);
      }
    }
    const uint4 ov = pack_bf16x8(acc);
    const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float lo = __uint_as_float(ow[i] << 16), hi = __uint_as_float(ow[i] & 0xFFFF0000u);
      ss = fmaf(lo, lo, ss);
      ss = fmaf(hi, hi, ss);
    }
    *reinterpret_cast<uint4*>(dst) = ov;
  }
  if (xhat_next && !out_f32) {
    __shared__ float red[kCombThreads / 32];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
    for (int i = 0; i < kCombThreads / 32; ++i) tot += red[i];
    const float r = 1.0f / sqrtf(tot / float(H) + 1e-6f);
    for (int h0 = threadIdx.x * VPT; h0 < H; h0 += kCombThreads * VPT) {
      const uint4 xv = *reinterpret_cast<const uint4*>(out + size_t(t) * H + h0);
      const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
      float hv[VPT];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        hv[2 * i] = __uint_as_float(xw[i] << 16) * r;
        hv[2 * i + 1] = __uint_as_float(xw[i] & 0xFFFF0000u) * r;
      }
      *reinterpret_cast<uint4*>(xhat_next + size_t(t) * H + h0) = pack_bf16x8(hv);
    }
  }
  pdl_launch_dependents();
}

}  // namespace

cudaError_t launch_combine(const LayerArgs& a) {
  const moe_config& c = a.cfg;
  return launch_pdl(a.y_half ? combine_kernel<true> : combine_kernel<false>, dim3(a.T), dim3(kCombThreads), 0,
                    a.stream, reinterpret_cast<const float*>(a.ws + a.L.y), reinterpret_cast<const int*>(a.ws + a.L.inv),
                    a.T, c.top_k, c.hidden, c.shared_inter > 0 ? 1 : 0, a.y, a.residual ? 1 : 0, a.xhat_next,
                    a.y_f32, a.gated ? reinterpret_cast<const int*>(a.ws + a.L.status) + ST_PATH : nullptr, a.x,
                    a.w.shared_gate_w);
}

}  // namespace moe
