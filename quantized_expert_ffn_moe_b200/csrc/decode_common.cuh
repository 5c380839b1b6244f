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

// Integer operands of the GEMV.  A code field shifted to the top of its byte
// and XOR-ed with 0x80 is, read as a signed byte, the code minus its offset
// times the field weight: for 4-bit codes c, ((c << 4) ^ 0x80) = 16 (c - 8);
// for 2-bit codes, ((c << 6) ^ 0x80) = 64 (c - 2).  The half-integer levels
// only change the constant: ((c << 4) ^ 0x88) = 16 (c - 7.5) and
// ((c << 6) ^ 0xA0) = 64 (c - 1.5).  dp2a multiplies two signed 16-bit
// activations with two of those bytes and adds them to a 32-bit sum, so a
// block's dot product is exact in int32 and is scaled once per block in fp32.
//
// The XOR constant of a format, one byte repeated.
__host__ __device__ inline uint32_t code_xor(int bits, int half_levels) {
  return half_levels ? (bits == 4 ? 0x88888888u : 0xA0A0A0A0u) : 0x80808080u;
}
// 4-bit word v = codes c0..c7 (c_j at bits 4j): returns the bytes
//   lo = (16 q0, 16 q2, 16 q4, 16 q6), hi = (16 q1, 16 q3, 16 q5, 16 q7)
__device__ __forceinline__ void q4_bytes(uint32_t v, uint32_t xk, uint32_t& lo, uint32_t& hi) {
  lo = lop_and_xor(v << 4, 0xF0F0F0F0u, xk);
  hi = lop_and_xor(v, 0xF0F0F0F0u, xk);
}
// 2-bit word v = codes c0..c15 (c_j at bits 2j): f[r] holds the bytes
// 64 q of elements r, r+4, r+8, r+12.
__device__ __forceinline__ void q2_bytes(uint32_t v, uint32_t xk, uint32_t (&f)[4]) {
  f[3] = lop_and_xor(v, 0xC0C0C0C0u, xk);
  f[2] = lop_and_xor(v << 2, 0xC0C0C0C0u, xk);
  f[1] = lop_and_xor(v << 4, 0xC0C0C0C0u, xk);
  f[0] = lop_and_xor(v << 6, 0xC0C0C0C0u, xk);
}
// Signed-byte weight of the code fields above: the dot products come out
// multiplied by 2^kCodeLog2.
template <int BITS> struct CodeMul { static constexpr int kLog2 = BITS == 4 ? 4 : 6; };

// Position, inside one code word's group of G elements, of element j in the
// operand order of the dp2a calls: 4-bit (x0 x2 x4 x6 x1 x3 x5 x7), 2-bit
// (x0 x4 x8 x12 x1 x5 x9 x13 x2 x6 x10 x14 x3 x7 x11 x15).
__host__ __device__ inline int dot_slot(int bits, int j) {
  return bits == 4 ? (j & 1) * 4 + (j >> 1) : (j & 3) * 4 + (j >> 2);
}
// Inverse of dot_slot: the element at operand position s.
__host__ __device__ inline int dot_elem(int bits, int s) {
  return bits == 4 ? (s & 3) * 2 + (s >> 2) : (s & 3) * 4 + (s >> 2);
}

// Per-row power-of-two scale of the integer activations: the largest |x|
// lands in [2^13, 2^14), so every element rounds to a value that fits int16
// with a bit to spare.  Returns the shift sh (x_int = rint(x * 2^sh)).
__device__ __forceinline__ int act_shift(float vmax) {
  if (!(vmax > 0.f)) return 0;
  int ex;
  frexpf(vmax, &ex);
  return min(max(14 - ex, -100), 100);
}
// Factor that turns a row's fp32 sum of (scale x integer dot) back into the
// real dot product: 2^-sh for the activations, 2^-kLog2 for the code bytes.
template <int BITS>
__device__ __forceinline__ float act_inv(int sh) { return ldexpf(1.f, -sh - CodeMul<BITS>::kLog2); }

// G consecutive activations (one code word's elements) times mul, rounded to
// int16 and packed in dot_slot order as G/8 16-byte parts, in registers.
template <int BITS, int G>
__device__ __forceinline__ void pack_int_order(const float (&v)[G], float mul, uint4 (&parts)[G / 8]) {
  uint32_t w[G / 2];
#pragma unroll
  for (int i = 0; i < G / 2; ++i) {
    const int a = __float2int_rn(v[dot_elem(BITS, 2 * i)] * mul);
    const int b = __float2int_rn(v[dot_elem(BITS, 2 * i + 1)] * mul);
    w[i] = (uint32_t(a) & 0xFFFFu) | (uint32_t(b) << 16);
  }
#pragma unroll
  for (int q = 0; q < G / 8; ++q) parts[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
}

// Offset (in 16-bit units) of element h of a staged activation row: the
// order in which a lane of a row group meets the operand pairs of its code
// words (dot_slot), laid out so that the lanes of a group read consecutive
// 16-byte slots.
template <int BITS, int LPR, int CPL>
__device__ __forceinline__ int staged_offset(int h) {
  using Gm = Geom<BITS, LPR, CPL>;
  const int c = h / Gm::W16, o = h % Gm::W16;
  const int s = c / LPR, lr = c % LPR;
  const int m = o / Gm::G, j = o % Gm::G;
  const int slot = dot_slot(BITS, j);
  const int part = slot >> 3, within = slot & 7;
  return ((((s * 4 + m) * Gm::NPART + part) * LPR + lr) << 3) + within;
}

// Value of an E4M3 byte (sign, 4 exponent bits with bias 7, 3 mantissa bits;
// exponent field 0 holds the subnormals m * 2^-9), exact in fp32.  The
// encoder never writes the two NaN codes (0x7F, 0xFF).
__device__ __forceinline__ float e4m3_value(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  const float mag = e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : float(m) * 0.001953125f;
  return (b & 0x80u) ? -mag : mag;
}

// Two E4M3 bytes (v & 0xFF, then (v >> 8) & 0xFF) to fp16 in one hardware
// conversion: every E4M3 value, subnormals included, is exact in fp16 (its
// smallest step 2^-9 and largest value 448 lie inside fp16's range), so the
// pair read as fp32 equals e4m3_value of each byte.
__device__ __forceinline__ __half2 e4m3x2_to_h2(uint32_t v) {
  uint32_t d;
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, lo;\n\t}" : "=r"(d) : "r"(v));
  return *reinterpret_cast<__half2*>(&d);
}

// Two rows of one stage (codes + scales in shared memory) and their row index
// in the expert matrix.  With fp8 block scales (SF = 1 below) a scale is one
// E4M3 byte and the rows carry their fp32 row scales rs0, rs1.
struct Rows {
  const unsigned char* codes;     // row rl0; row rl0+1 follows at +RB
  const unsigned char* scales;    // row rl0; row rl0+1 follows at +(SPR >> PS) scales
  int r0;
  uint32_t xk;                    // code_xor of the format
  float rs0 = 1.f, rs1 = 1.f;     // fp8 block scales only: the rows' fp32 scales
};

// Scales per row, and the piece-to-scale shift PS of a 4-bit block of 32
// (PS 0) or 128 (PS 2): the 32-element piece c takes scale c >> PS.  2-bit:
// blocks of 16, four per 64-element piece, PS 0.
__host__ __device__ inline int scales_per_row(int K, int block) { return K / block; }
__host__ __device__ inline int piece_shift(int bits, int block) { return bits == 4 && block == 128 ? 2 : 0; }

// Dot products of the lane group's two rows with NT staged tokens, reduced
// over the LPR lanes of the row, then the epilogue.  Per code word the lane
// turns the codes into signed bytes (q4_bytes / q2_bytes) and runs dp2a
// against the int16 activations (two independent int32 chains per row and
// token); each block's exact integer sum is converted to fp32 and multiplied
// by the block's scale (fp16, or with SF = 1 an E4M3 byte, the row's fp32
// scale then applied once per output).  `nt` <= NT tokens are valid; xs holds
// int16 activations staged with staged_offset.
template <int MODE, int BITS, int LPR, int CPL, int NT, int PS = 0, int SF = 0>
__device__ __forceinline__ void rows_dot(float* out, int out_cols, const Rows& rw, const int16_t* xs, int tb, int lr,
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
      if (SF) {                                   // both rows' scale bytes in one conversion
        const float2 f = __half22float2(e4m3x2_to_h2(uint32_t(rw.scales[c >> PS]) |
                                                     (uint32_t(rw.scales[(Gm::SPR >> PS) + (c >> PS)]) << 8)));
        sc[0] = f.x;
        sc[1] = f.y;
      } else {
#pragma unroll
        for (int rho = 0; rho < 2; ++rho)
          sc[rho] = __half2float(*reinterpret_cast<const __half*>(rw.scales + rho * (Gm::SPR >> PS) * 2 + (c >> PS) * 2));
      }
      int ia[2][NT], ib[2][NT];
#pragma unroll
      for (int rho = 0; rho < 2; ++rho)
#pragma unroll
        for (int t = 0; t < NT; ++t) ia[rho][t] = ib[rho][t] = 0;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        uint32_t lo[2], hi[2];
        q4_bytes(wd[0][m], rw.xk, lo[0], hi[0]);
        q4_bytes(wd[1][m], rw.xk, lo[1], hi[1]);
        const int xoff = ((s * 4 + m) * LPR + lr) * 8;
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const uint4 xv = *reinterpret_cast<const uint4*>(xs + xr0[t] + xoff);
#pragma unroll
          for (int rho = 0; rho < 2; ++rho) {
            ia[rho][t] = __dp2a_lo(int(xv.x), int(lo[rho]), ia[rho][t]);
            ib[rho][t] = __dp2a_hi(int(xv.y), int(lo[rho]), ib[rho][t]);
            ia[rho][t] = __dp2a_lo(int(xv.z), int(hi[rho]), ia[rho][t]);
            ib[rho][t] = __dp2a_hi(int(xv.w), int(hi[rho]), ib[rho][t]);
          }
        }
      }
#pragma unroll
      for (int rho = 0; rho < 2; ++rho)
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[rho][t] = fmaf(sc[rho], __int2float_rn(ia[rho][t] + ib[rho][t]), acc[rho][t]);
    } else {
      // the four scales of the piece's blocks as four fp16: read (8 bytes), or
      // converted from four E4M3 bytes
      uint2 scp[2];
#pragma unroll
      for (int rho = 0; rho < 2; ++rho) {
        if (SF) {
          const uint32_t b4 = *reinterpret_cast<const uint32_t*>(rw.scales + rho * Gm::SPR + c * 4);
          const __half2 h01 = e4m3x2_to_h2(b4), h23 = e4m3x2_to_h2(b4 >> 16);
          scp[rho] = make_uint2(*reinterpret_cast<const uint32_t*>(&h01), *reinterpret_cast<const uint32_t*>(&h23));
        } else {
          scp[rho] = *reinterpret_cast<const uint2*>(rw.scales + rho * Gm::SPR * 2 + c * 8);
        }
      }
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        uint32_t f[2][4];
        q2_bytes(wd[0][m], rw.xk, f[0]);
        q2_bytes(wd[1][m], rw.xk, f[1]);
        const int xoff = ((s * 4 + m) * 2 * LPR + lr) * 8;
        float sc[2];
#pragma unroll
        for (int rho = 0; rho < 2; ++rho) {
          const uint32_t pr = (m < 2) ? scp[rho].x : scp[rho].y;
          sc[rho] = __half2float(__ushort_as_half((unsigned short)((m & 1) ? (pr >> 16) : (pr & 0xFFFFu))));
        }
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const int16_t* xr = xs + xr0[t] + xoff;
          const uint4 xa = *reinterpret_cast<const uint4*>(xr);
          const uint4 xb = *reinterpret_cast<const uint4*>(xr + LPR * 8);
#pragma unroll
          for (int rho = 0; rho < 2; ++rho) {
            int ia = __dp2a_lo(int(xa.x), int(f[rho][0]), 0);
            int ib = __dp2a_hi(int(xa.y), int(f[rho][0]), 0);
            ia = __dp2a_lo(int(xa.z), int(f[rho][1]), ia);
            ib = __dp2a_hi(int(xa.w), int(f[rho][1]), ib);
            ia = __dp2a_lo(int(xb.x), int(f[rho][2]), ia);
            ib = __dp2a_hi(int(xb.y), int(f[rho][2]), ib);
            ia = __dp2a_lo(int(xb.z), int(f[rho][3]), ia);
            ib = __dp2a_hi(int(xb.w), int(f[rho][3]), ib);
            acc[rho][t] = fmaf(sc[rho], __int2float_rn(ia + ib), acc[rho][t]);
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
        float g = acc[0][t] * inv, u = acc[1][t] * inv;
        if (SF) { g *= rw.rs0; u *= rw.rs1; }
        out[size_t(p) * out_cols + (rw.r0 >> 1)] = g / (1.f + expf(-g)) * u;
      } else {
        const float wgt = tok_w[tl] * inv;
        float y0 = acc[0][t] * wgt, y1 = acc[1][t] * wgt;
        if (SF) { y0 *= rw.rs0; y1 *= rw.rs1; }
        *reinterpret_cast<float2*>(out + size_t(p) * out_cols + rw.r0) = make_float2(y0, y1);
      }
    }
  }
}

}  // namespace gemv
}  // namespace moe
