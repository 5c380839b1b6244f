// Device side of the seeded input generator (libmoe_inputs.so).  Same recipe
// as moe_inputs/gen.py, using only integer arithmetic and single correctly
// rounded fp32 operations so that both sides produce identical bytes:
//   SplitMix64 output function as a counter-based hash, Irwin-Hall sum of the
//   four 16-bit fields as an approximate normal deviate, fp32 masters, and the
//   symmetric absmax block encoder of the packed weight format.
// This library prepares inputs only; it is not part of the MoE layer.
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace {

constexpr uint64_t kGolden = 0x9E3779B97F4A7C15ull;
enum { ROLE_ROUTER = 0, ROLE_GATE = 1, ROLE_UP = 2, ROLE_DOWN = 3, ROLE_SH_GATE = 4, ROLE_SH_UP = 5,
       ROLE_SH_DOWN = 6 };

__host__ __device__ inline uint64_t mix64(uint64_t z) {
  z ^= z >> 30;
  z *= 0xBF58476D1CE4E5B9ull;
  z ^= z >> 27;
  z *= 0x94D049BB133111EBull;
  z ^= z >> 31;
  return z;
}

__host__ __device__ inline uint64_t stream_key(uint64_t seed, uint64_t layer, uint64_t role, uint64_t expert) {
  uint64_t k = mix64(seed);
  k = mix64(k + layer);
  k = mix64(k + role);
  k = mix64(k + expert);
  return k;
}

__device__ inline float normal_at(uint64_t key, uint64_t i, float c) {
  const uint64_t z = mix64(key + (i + 1) * kGolden);
  const int s = int(z & 0xFFFF) + int((z >> 16) & 0xFFFF) + int((z >> 32) & 0xFFFF) + int(z >> 48);
  const int d = 2 * s - 262140;
  return __fmul_rn(float(d), c);
}

struct PoolArgs {
  uint64_t seed;
  int layer, E, H, I, bits, block;
  int e0, ne, shared, half;
  float c;
  uint8_t* gu_codes;
  uint16_t* gu_scales;
  uint8_t* d_codes;
  uint16_t* d_scales;
};

// One thread per quantisation block.
__global__ void gen_pool_kernel(PoolArgs a) {
  const long long gu_blocks = (long long)2 * a.I * (a.H / a.block);
  const long long d_blocks = (long long)a.H * (a.I / a.block);
  const long long per_expert = gu_blocks + d_blocks;
  const long long total = per_expert * a.ne;
  const int qmax = (1 << (a.bits - 1)) - 1;
  for (long long tid = blockIdx.x * (long long)blockDim.x + threadIdx.x; tid < total;
       tid += (long long)gridDim.x * blockDim.x) {
    const int slot = int(tid / per_expert);
    long long b = tid % per_expert;
    const int expert = a.shared ? 0 : a.e0 + slot;
    int role, row, col0, K;
    bool is_gu = b < gu_blocks;
    int packed_row;
    if (is_gu) {
      const int bpr = a.H / a.block;
      packed_row = int(b / bpr);
      col0 = int(b % bpr) * a.block;
      row = packed_row >> 1;
      role = (packed_row & 1) ? (a.shared ? ROLE_SH_UP : ROLE_UP) : (a.shared ? ROLE_SH_GATE : ROLE_GATE);
      K = a.H;
    } else {
      b -= gu_blocks;
      const int bpr = a.I / a.block;
      packed_row = int(b / bpr);
      col0 = int(b % bpr) * a.block;
      row = packed_row;
      role = a.shared ? ROLE_SH_DOWN : ROLE_DOWN;
      K = a.I;
    }
    const uint64_t key = stream_key(a.seed, (uint64_t)a.layer, (uint64_t)role, (uint64_t)expert);
    float w[128];                        // block <= 128 elements
    float amax = 0.f;
    for (int j = 0; j < a.block; ++j) {
      w[j] = normal_at(key, (uint64_t)row * K + col0 + j, a.c);
      amax = fmaxf(amax, fabsf(w[j]));
    }
    // half-integer levels: top level qmax + 1/2, code of the level just
    // above w / s (floor + 2^(bits-1)), clamped to the 2^bits codes
    const float top = a.half ? float(qmax) + 0.5f : float(qmax);
    const __half s16 = __float2half_rn(__fdiv_rn(amax, top));
    const float sf = __half2float(s16);
    uint32_t packed[16] = {0};           // up to 64 bytes of codes per block
    for (int j = 0; j < a.block; ++j) {
      int code = 1 << (a.bits - 1);
      if (sf != 0.f) {
        const float ratio = __fdiv_rn(w[j], sf);
        if (a.half) {
          code = int(floorf(ratio)) + (1 << (a.bits - 1));
          code = code < 0 ? 0 : (code > (1 << a.bits) - 1 ? (1 << a.bits) - 1 : code);
        } else {
          int q = int(rintf(ratio));
          q = q < -qmax ? -qmax : (q > qmax ? qmax : q);
          code = q + (1 << (a.bits - 1));
        }
      }
      const int bit = j * a.bits;
      packed[bit >> 5] |= uint32_t(code) << (bit & 31);
    }
    const int code_bytes = a.block * a.bits / 8;
    const size_t row_bytes = size_t(K) * a.bits / 8;
    uint8_t* cdst;
    uint16_t* sdst;
    if (is_gu) {
      cdst = a.gu_codes + size_t(slot) * 2 * a.I * (size_t(a.H) * a.bits / 8) + size_t(packed_row) * row_bytes;
      sdst = a.gu_scales + size_t(slot) * 2 * a.I * (a.H / a.block) + size_t(packed_row) * (K / a.block);
    } else {
      cdst = a.d_codes + size_t(slot) * a.H * (size_t(a.I) * a.bits / 8) + size_t(packed_row) * row_bytes;
      sdst = a.d_scales + size_t(slot) * a.H * (a.I / a.block) + size_t(packed_row) * (K / a.block);
    }
    cdst += size_t(col0) * a.bits / 8;
    for (int q = 0; q < code_bytes / 4; ++q) reinterpret_cast<uint32_t*>(cdst)[q] = packed[q];
    sdst[col0 / a.block] = __half_as_ushort(s16);
  }
}

// E4M3 byte nearest to a non-negative fp32 value (ties to even, saturating at
// 448; exponent field 0 holds the subnormals m * 2^-9), and the value of a
// non-negative byte: the encoder of moe_inputs.gen.e4m3_encode, step for step.
__device__ inline uint32_t e4m3_encode(float t) {
  if (t < 0.015625f) return uint32_t(rintf(__fmul_rn(t, 512.f)));       // 8 -> code 8 = 2^-6
  const uint32_t bits = __float_as_uint(t);
  int e = int(bits >> 23) - 127;
  const float mant = __uint_as_float((bits & 0x7FFFFFu) | 0x3F800000u);  // t / 2^e in [1, 2)
  int m = int(rintf(__fmul_rn(__fsub_rn(mant, 1.f), 8.f)));
  if (m == 8) { ++e; m = 0; }
  const int code = ((e + 7) << 3) | m;
  return uint32_t(code < 0x7E ? code : 0x7E);
}
__device__ inline float e4m3_nonneg_value(uint32_t code) {
  const uint32_t e = (code >> 3) & 15u, m = code & 7u;
  return e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : float(m) * 0.001953125f;
}

struct PoolF8Args {
  uint64_t seed;
  int layer, E, H, I, bits, block;
  int e0, ne, shared;
  float c;
  uint8_t* gu_codes;
  uint8_t* gu_scales;
  uint8_t* d_codes;
  uint8_t* d_scales;
  float* gu_rs;
  float* d_rs;
};

// One warp per weight row: the row's block maxima, the row scale
// S = rowmax / (qmax * 448), one E4M3 byte per block for blockmax / (qmax S),
// then the integer codes against e4m3 * S (quantize_blocks_e4m3 of the host
// generator).  Blocks of up to 32 elements; up to 8 blocks per lane.
__global__ void gen_pool_f8_kernel(PoolF8Args a) {
  const int lane = threadIdx.x & 31;
  const long long rows_per_expert = 2LL * a.I + a.H;
  const long long total = rows_per_expert * a.ne;
  const int qmax = (1 << (a.bits - 1)) - 1;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long wr = blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5); wr < total; wr += warps) {
    const int slot = int(wr / rows_per_expert);
    int prow = int(wr % rows_per_expert);
    const int expert = a.shared ? 0 : a.e0 + slot;
    const bool is_gu = prow < 2 * a.I;
    int role, row, K;
    if (is_gu) {
      row = prow >> 1;
      role = (prow & 1) ? (a.shared ? ROLE_SH_UP : ROLE_UP) : (a.shared ? ROLE_SH_GATE : ROLE_GATE);
      K = a.H;
    } else {
      prow -= 2 * a.I;
      row = prow;
      role = a.shared ? ROLE_SH_DOWN : ROLE_DOWN;
      K = a.I;
    }
    const uint64_t key = stream_key(a.seed, (uint64_t)a.layer, (uint64_t)role, (uint64_t)expert);
    const int nb = K / a.block;
    float am[8];
    float rmax = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      am[k] = 0.f;
      const int b = lane + 32 * k;
      if (b < nb) {
        for (int j = 0; j < a.block; ++j)
          am[k] = fmaxf(am[k], fabsf(normal_at(key, (uint64_t)row * K + b * a.block + j, a.c)));
        rmax = fmaxf(rmax, am[k]);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) rmax = fmaxf(rmax, __shfl_xor_sync(0xffffffffu, rmax, o));
    const float S = __fdiv_rn(rmax, float(qmax * 448));
    const float den = __fmul_rn(S, float(qmax));
    uint8_t* cdst;
    uint8_t* sdst;
    if (is_gu) {
      cdst = a.gu_codes + size_t(slot) * 2 * a.I * (size_t(a.H) * a.bits / 8) + size_t(prow) * (size_t(K) * a.bits / 8);
      sdst = a.gu_scales + size_t(slot) * 2 * a.I * (a.H / a.block) + size_t(prow) * nb;
      if (lane == 0) a.gu_rs[size_t(slot) * 2 * a.I + prow] = S;
    } else {
      cdst = a.d_codes + size_t(slot) * a.H * (size_t(a.I) * a.bits / 8) + size_t(prow) * (size_t(K) * a.bits / 8);
      sdst = a.d_scales + size_t(slot) * a.H * (a.I / a.block) + size_t(prow) * nb;
      if (lane == 0) a.d_rs[size_t(slot) * a.H + prow] = S;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int b = lane + 32 * k;
      if (b >= nb) continue;
      const uint32_t s8 = den > 0.f ? e4m3_encode(__fdiv_rn(am[k], den)) : 0u;
      const float sf = __fmul_rn(e4m3_nonneg_value(s8), S);
      uint32_t packed[4] = {0u, 0u, 0u, 0u};   // 16 bytes of codes per 4-bit block of 32, 4 per 2-bit block of 16
      for (int j = 0; j < a.block; ++j) {
        int q = 0;
        if (sf != 0.f) {
          q = int(rintf(__fdiv_rn(normal_at(key, (uint64_t)row * K + b * a.block + j, a.c), sf)));
          q = q < -qmax ? -qmax : (q > qmax ? qmax : q);
        }
        const int bit = j * a.bits;
        packed[bit >> 5] |= uint32_t(q + (1 << (a.bits - 1))) << (bit & 31);
      }
      const int code_bytes = a.block * a.bits / 8;
      uint8_t* cb = cdst + size_t(b) * code_bytes;
      for (int q = 0; q < code_bytes / 4; ++q) reinterpret_cast<uint32_t*>(cb)[q] = packed[q];
      sdst[b] = uint8_t(s8);
    }
  }
}

__global__ void gen_bf16_kernel(uint64_t key, uint64_t start, uint64_t n, float c, uint16_t* out) {
  for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < n; i += (uint64_t)gridDim.x * blockDim.x) {
    const __nv_bfloat16 b = __float2bfloat16_rn(normal_at(key, start + i, c));
    out[i] = __bfloat16_as_ushort(b);
  }
}

}  // namespace

extern "C" {

// Packed pool of experts [e0, e0+ne) of one layer (shared == 0), or of the
// shared expert (shared == 1, ne == 1).  Outputs are device buffers laid out
// as in include/moe_capi.h, starting at the first generated expert.
// c = fp32 sigma / 75674.45 (bits 0x348de3bd for sigma 0.02).
int moe_gen_pool(uint64_t seed, int layer, int E, int H, int I, int bits, int block, int half, int e0, int ne,
                 int shared, float c, uint8_t* gu_codes, uint16_t* gu_scales, uint8_t* d_codes, uint16_t* d_scales,
                 void* stream) {
  if (!((bits == 4 && (block == 32 || block == 128)) || (bits == 2 && block == 16))) return -2;
  if (ne <= 0 || (shared && ne != 1) || (!shared && (e0 < 0 || e0 + ne > E))) return -1;
  if (!gu_codes || !gu_scales || !d_codes || !d_scales) return -1;
  if (H % block || I % block) return -2;
  PoolArgs a{(uint64_t)seed, layer, E, H, I, bits, block, e0, ne, shared, half ? 1 : 0, c, gu_codes, gu_scales,
             d_codes, d_scales};
  gen_pool_kernel<<<148 * 16, 256, 0, static_cast<cudaStream_t>(stream)>>>(a);
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

// The same pool with one E4M3 scale byte per block (4-bit blocks of 32, 2-bit
// blocks of 16) and one fp32 scale per row (gu_rs [ne][2I], d_rs [ne][H]).
int moe_gen_pool_f8(uint64_t seed, int layer, int E, int H, int I, int bits, int block, int e0, int ne, int shared,
                    float c, uint8_t* gu_codes, uint8_t* gu_scales, uint8_t* d_codes, uint8_t* d_scales, float* gu_rs,
                    float* d_rs, void* stream) {
  if (!((bits == 4 && block == 32) || (bits == 2 && block == 16))) return -2;
  if (ne <= 0 || (shared && ne != 1) || (!shared && (e0 < 0 || e0 + ne > E))) return -1;
  if (!gu_codes || !gu_scales || !d_codes || !d_scales || !gu_rs || !d_rs) return -1;
  if (H % block || I % block || H / block > 256 || I / block > 256) return -2;
  PoolF8Args a{(uint64_t)seed, layer, E, H, I, bits, block, e0, ne, shared, c, gu_codes, gu_scales, d_codes, d_scales,
               gu_rs, d_rs};
  gen_pool_f8_kernel<<<148 * 8, 256, 0, static_cast<cudaStream_t>(stream)>>>(a);
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

// n bf16 values N(0, sigma) of stream `key`, elements start .. start+n-1.
int moe_gen_normal_bf16(uint64_t key, uint64_t start, uint64_t n, float c, uint16_t* out, void* stream) {
  if (!out) return -1;
  if (n == 0) return 0;
  gen_bf16_kernel<<<148 * 8, 256, 0, static_cast<cudaStream_t>(stream)>>>(key, start, n, c, out);
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

uint64_t moe_gen_stream_key(uint64_t seed, int layer, int role, int expert) {
  return stream_key(seed, (uint64_t)layer, (uint64_t)role, (uint64_t)expert);
}

}  // extern "C"
