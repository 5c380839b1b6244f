// Building blocks of the decode GEMV shared by the standalone pass kernels
// (decode.cu) and the fused decode kernel (fused.cu).
#pragma once

#include "moe_internal.cuh"

namespace moe {
namespace gemv {

constexpr int kNCW = 8;                     // consumer warps
constexpr int kThreads = (kNCW + 1) * 32;   // + one producer warp
constexpr int kStages = 4;                  // shared-memory ring depth
constexpr int kSmemBudget = 220 * 1024;
constexpr int kMaxNTC = 64;

enum Mode { GATEUP = 0, DOWN = 1 };

template <int BITS, int LPR, int CPL>
struct Geom {
  static constexpr int RW = 32 / LPR;                 // lane groups (row pairs) per warp
  static constexpr int W16 = BITS == 4 ? 32 : 64;     // weights per 16-byte piece
  static constexpr int K = LPR * CPL * W16;           // reduction length
  static constexpr int NPART = BITS == 4 ? 1 : 2;     // 16-byte activation slots per code word
  static constexpr int G = BITS == 4 ? 8 : 16;        // elements per code word
  static constexpr int BLOCK = BITS == 4 ? 32 : 16;  // smallest block of the format (4-bit also runs 128)
  static constexpr int SPR = K / BLOCK;               // scales per row at that block (stage upper bound)
  static constexpr int RB = K * BITS / 8;             // code bytes per row
  static constexpr int RPS = kNCW * RW * 2;           // rows per pipeline stage
  static constexpr int CODE_BYTES = RPS * RB;
  static constexpr int SCALE_BYTES = RPS * SPR * 2;
  static constexpr int STAGE_BYTES = (CODE_BYTES + SCALE_BYTES + 127) / 128 * 128;
};

// Offset (in halves) of element h of a staged activation row: the order in
// which a lane of a row group meets the decoded half2 pairs (see decode_q4x8 /
// decode_q2x16), laid out so that the lanes of a group read consecutive
// 16-byte slots.
template <int BITS, int LPR, int CPL>
__device__ __forceinline__ int staged_offset(int h) {
  using Gm = Geom<BITS, LPR, CPL>;
  const int c = h / Gm::W16, o = h % Gm::W16;
  const int s = c / LPR, lr = c % LPR;
  const int m = o / Gm::G, j = o % Gm::G;
  const int slot = decode_slot(BITS, j);
  const int part = slot >> 3, within = slot & 7;
  return ((((s * 4 + m) * Gm::NPART + part) * LPR + lr) << 3) + within;
}

// Two rows of one stage (codes + scales in shared memory) and their row index
// in the expert matrix.
struct Rows {
  const unsigned char* codes;     // row rl0; row rl0+1 follows at +RB
  const unsigned char* scales;    // row rl0; row rl0+1 follows at +(SPR >> PS)*2
  int r0;
};

// Scales per row, and the piece-to-scale shift PS of a 4-bit block of 32
// (PS 0) or 128 (PS 2): the 32-element piece c takes scale c >> PS.  2-bit:
// blocks of 16, four per 64-element piece, PS 0.
__host__ __device__ inline int scales_per_row(int K, int block) { return K / block; }
__host__ __device__ inline int piece_shift(int bits, int block) { return bits == 4 && block == 128 ? 2 : 0; }

// Dot products of the lane group's two rows with NT staged tokens, reduced
// over the LPR lanes of the row, then the epilogue.  Each block's products
// accumulate in two independent fp16x2 chains (even / odd code words) and
// are folded into fp32 with the block scale.  `nt` <= NT tokens are valid.
template <int MODE, int BITS, int LPR, int CPL, int NT, int PS = 0>
__device__ __forceinline__ void rows_dot(float* out, int out_cols, const Rows& rw, const __half* xs, int tb, int lr,
                                         const float* tok_inv, const float* tok_w, const int* tok_pos,
                                         int nt = NT, const int* xrow = nullptr) {
  using Gm = Geom<BITS, LPR, CPL>;
  constexpr int K = Gm::K;
  // staged activation row of each token of the block: consecutive rows after
  // xs, or the rows listed in xrow (activations staged once per token).  Token
  // slots past nt repeat the first token, so the inner loops run branch-free
  // and only the epilogue skips them.
  int xr0[NT];
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int tt = t < nt ? t : 0;
    xr0[t] = (xrow ? xrow[tb + tt] : tt) * K;
  }
  float acc[2][NT];
#pragma unroll
  for (int rho = 0; rho < 2; ++rho)
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[rho][t] = 0.f;
#pragma unroll
  for (int s = 0; s < CPL; ++s) {
    const int c = s * LPR + lr;
    const uint4 cw0 = *reinterpret_cast<const uint4*>(rw.codes + c * 16);
    const uint4 cw1 = *reinterpret_cast<const uint4*>(rw.codes + Gm::RB + c * 16);
    const uint32_t wd[2][4] = {{cw0.x, cw0.y, cw0.z, cw0.w}, {cw1.x, cw1.y, cw1.z, cw1.w}};
    if (BITS == 4) {
      float sc[2];
#pragma unroll
      for (int rho = 0; rho < 2; ++rho)
        sc[rho] = __half2float(*reinterpret_cast<const __half*>(rw.scales + rho * (Gm::SPR >> PS) * 2 + (c >> PS) * 2));
      __half2 hacc[2][NT][2];
#pragma unroll
      for (int rho = 0; rho < 2; ++rho)
#pragma unroll
        for (int t = 0; t < NT; ++t) hacc[rho][t][0] = hacc[rho][t][1] = __float2half2_rn(0.f);
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        __half2 q[2][4];
        decode_q4x8(wd[0][m], q[0]);
        decode_q4x8(wd[1][m], q[1]);
        const int xoff = ((s * 4 + m) * LPR + lr) * 8;
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const uint4 xv = *reinterpret_cast<const uint4*>(xs + xr0[t] + xoff);
          const __half2 x2[4] = {u32_as_h2(xv.x), u32_as_h2(xv.y), u32_as_h2(xv.z), u32_as_h2(xv.w)};
#pragma unroll
          for (int rho = 0; rho < 2; ++rho)
#pragma unroll
            for (int z = 0; z < 4; ++z) hacc[rho][t][m & 1] = __hfma2(q[rho][z], x2[z], hacc[rho][t][m & 1]);
        }
      }
#pragma unroll
      for (int rho = 0; rho < 2; ++rho)
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const float2 f = __half22float2(__hadd2(hacc[rho][t][0], hacc[rho][t][1]));
          acc[rho][t] = fmaf(sc[rho], f.x + f.y, acc[rho][t]);
        }
    } else {
      uint2 scp[2];
#pragma unroll
      for (int rho = 0; rho < 2; ++rho) scp[rho] = *reinterpret_cast<const uint2*>(rw.scales + rho * Gm::SPR * 2 + c * 8);
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        __half2 q[2][8];
        decode_q2x16(wd[0][m], q[0]);
        decode_q2x16(wd[1][m], q[1]);
        const int xoff = ((s * 4 + m) * 2 * LPR + lr) * 8;
        float sc[2];
#pragma unroll
        for (int rho = 0; rho < 2; ++rho) {
          const uint32_t pr = (m < 2) ? scp[rho].x : scp[rho].y;
          sc[rho] = __half2float(__ushort_as_half((unsigned short)((m & 1) ? (pr >> 16) : (pr & 0xFFFFu))));
        }
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const __half* xr = xs + xr0[t] + xoff;
          const uint4 xa = *reinterpret_cast<const uint4*>(xr);
          const uint4 xb = *reinterpret_cast<const uint4*>(xr + LPR * 8);
          const __half2 x2[8] = {u32_as_h2(xa.x), u32_as_h2(xa.y), u32_as_h2(xa.z), u32_as_h2(xa.w),
                                 u32_as_h2(xb.x), u32_as_h2(xb.y), u32_as_h2(xb.z), u32_as_h2(xb.w)};
#pragma unroll
          for (int rho = 0; rho < 2; ++rho) {
            __half2 h0 = __hmul2(q[rho][0], x2[0]), h1 = __hmul2(q[rho][1], x2[1]);
#pragma unroll
            for (int z = 2; z < 8; z += 2) {
              h0 = __hfma2(q[rho][z], x2[z], h0);
              h1 = __hfma2(q[rho][z + 1], x2[z + 1], h1);
            }
            const float2 f = __half22float2(__hadd2(h0, h1));
            acc[rho][t] = fmaf(sc[rho], f.x + f.y, acc[rho][t]);
          }
        }
      }
    }
  }
  // reduce across the LPR lanes of each row
#pragma unroll
  for (int t = 0; t < NT; ++t) {
#pragma unroll
    for (int rho = 0; rho < 2; ++rho)
#pragma unroll
      for (int o = LPR / 2; o > 0; o >>= 1) acc[rho][t] += __shfl_xor_sync(0xffffffffu, acc[rho][t], o);
  }
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int tl = tb + t;
    if (t < nt && lr == (t % LPR)) {
      const float inv = tok_inv[tl];
      const int p = tok_pos[tl];
      if (MODE == GATEUP) {
        const float g = acc[0][t] * inv, u = acc[1][t] * inv;
        out[size_t(p) * out_cols + (rw.r0 >> 1)] = g / (1.f + expf(-g)) * u;
      } else {
        const float wgt = tok_w[tl] * inv;
        *reinterpret_cast<float2*>(out + size_t(p) * out_cols + rw.r0) = make_float2(acc[0][t] * wgt, acc[1][t] * wgt);
      }
    }
  }
}

}  // namespace gemv
}  // namespace moe
