// Fused decode: a whole MoE layer -- or a stack of layers -- for a small batch
// in one cooperative launch of one CTA per SM.
//
// Same operation as the separate kernels (router logits, top-k with
// renormalised gates, grouping, gate/up + SwiGLU, down, gate-weighted combine
// with the shared expert; in the stack RMSNorm before and the bf16 residual
// after each layer), reorganised so that a decode step pays one launch:
//
//   R  every CTA: stages the T tokens (RMSNorm factor in the stack, xhat as
//      int16 with a power-of-two scale) and computes the router logits of its
//      slice of experts -> global; the producer thread prefetches this CTA's
//      share of the shared expert's bytes into L2                 | grid barrier
//   S  every CTA (the same deterministic computation): top-k, gates, stable
//      grouping and the cost-balanced work lists, in shared memory
//   G  gate/up + SwiGLU over the CTA's share of the stages; the producer warp
//      streams them (1-D TMA bulk copies into a 4-slot ring) and runs straight
//      on into the CTA's down-pass stages                        | grid barrier
//   D  down x gate weight -> Y                                   | grid barrier
//   C  combine of the CTA's slice of (token, 8 columns) units    | grid barrier
//                                                                  (stack only)
// The consumers are two groups of 8 warps that take the stages alternately
// (group = stage index mod 2), so one group decodes while the other waits for
// its next stage.  A ring slot always belongs to the same group: with slots
// shared between groups a group could wait on a slot's barrier two phases
// ahead, where the parity test passes on the stale phase.
// Grid barriers: one word per launch, flipped by the last arrival; every spin
// is bounded (kWaitLimitCycles, then MOE_ERR_TIMEOUT in the status word and
// the CTA skips the rest).
// Decode is bound by moving expert weights ("125 billion parameters on one
// gaming GPU -- first impressions of Strata + Qwen 3.8 Flash Next", section "In
// brief": compute isn't the blocker); with one launch the HBM stream is not
// interrupted by kernel boundaries.
#include "decode_common.cuh"

namespace moe {

namespace {

using namespace gemv;

constexpr int kFGroups = 2;                       // consumer groups of kNCW warps
constexpr int kFCons = kFGroups * kNCW;           // consumer warps
constexpr int kFThreads = (kFCons + 1) * 32;      // + the producer warp
constexpr int kFStages = 4;                       // ring slots; slot s belongs to group s % kFGroups
static_assert(kFStages % kFGroups == 0, "a ring slot must belong to one consumer group");
constexpr int kBarAll = 1;                        // named barrier of all consumer warps (group g: 2 + g)
constexpr int kFRingOff = 3584;                   // shared-memory offset of the ring
constexpr int kFMaxTokens = 64;
constexpr int kFMaxPairs = kFMaxTokens * 16;
constexpr int kMaxFusedLayers = 64;
constexpr int kTimePoints = 32;

struct FusedParams {
  moe_config cfg;
  int T, L;
  int stack;                     // 1: x_inout residual stream with RMSNorm; 0: y = layer(x)
  const uint16_t* x;             // layer mode input
  uint16_t* y;                   // layer mode output, or the residual stream (stack)
  int* trace;                    // stack: [L][T][k] selections, or null
  unsigned long long* timing;    // null, or [gridDim][32] timestamps of layer 0 (moe_debug_fused_timing)
  char* ws;
  Layout L_;
  int ntc_gu, ntc_dn;             // tokens per chunk (gate/up: T when every token is pre-staged)
  int pre;                        // 1: all T tokens staged once per layer for the router and gate/up
  int rtc;                        // router: tokens staged at a time
  int grp_xs;                     // halves of one group's chunk buffer
  long long xs_halves;            // halves of the whole token region
  int smem_route_off, smem_xs_off;
  // single layer, 32..64 tokens: after routing, hand the layer to the grouped
  // tcgen05 kernels that follow in the stream when their predicted time is
  // lower (hybrid 1 = choose, 2 = always hand over)
  int hybrid;
  float cost_f0, cost_f1;         // CUDA-core time model: f0 + f1 * cost units per CTA (us)
  float cost_t0, cost_t1;         // tensor-core time model: t0 + t1 * k-blocks per CTA (us)
  moe_layer_weights w[kMaxFusedLayers];
};

// ------------------------------------------------------------ grid barrier
// One thread per CTA, after a CTA-wide barrier.  CTA 0 adds 2^31 - (G - 1),
// the others 1, so the word's top bit flips exactly when the last CTA
// arrives and the low bits return to zero (the word starts at zero in every
// launch); each CTA waits for the flip of the value its own add returned.
// Returns false when the wait gave up.
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ unsigned atom_add_release_u32(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.add.release.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

__device__ bool grid_barrier(unsigned* word, unsigned nblocks, int* status) {
  const unsigned inc = blockIdx.x == 0 ? 0x80000000u - (nblocks - 1u) : 1u;
  __threadfence();
  const unsigned old = atom_add_release_u32(word, inc);
  const long long t0 = clock64();
  while (((ld_acquire_u32(word) ^ old) & 0x80000000u) == 0u) {
    if (clock64() - t0 > kWaitLimitCycles) {
      report_error(status, MOE_ERR_TIMEOUT, 40);
      return false;
    }
  }
  __threadfence();
  return true;
}

// Routing of the current layer, one copy per CTA in shared memory.
struct SRoute {
  int* idx;      // [T*k]
  float* w;      // [T*k]
  int* pairs;    // [T*k] pair id at each routed position
  int* inv;      // [T*k] position of each pair
  int* offsets;  // [E+1]
  int* ulist;    // [E+1]
  int* woff_gu;  // [E+2]
  int* woff_dn;  // [E+2]
  unsigned* tmask;  // [ceil(T/32)][E] tokens that picked each expert (bit t % 32)
};

// Cursor over a CTA's stages in shared-memory routing (same walk as the
// standalone GEMV's cursor).
struct FCursor {
  const SRoute* r;
  int T, k, E, spe, ntc;
  int slot, n, p0, e, chunk, nc, stage;
  long long pos;
  const int* woff;
  int nslots;

  __device__ void range(int s, int* e_, int* p0_, int* n_) const {
    const int ee = r->ulist[s];
    *e_ = ee;
    if (ee >= E) { *p0_ = T * k; *n_ = T; }
    else { *p0_ = r->offsets[ee]; *n_ = r->offsets[ee + 1] - r->offsets[ee]; }
  }
  __device__ void load_slot() {
    range(slot, &e, &p0, &n);
    chunk = 0;
    nc = min(ntc, n);
    stage = 0;
  }
  __device__ void next_chunk() {
    ++chunk;
    stage = 0;
    if (chunk * ntc >= n) {
      if (++slot < nslots) load_slot();
    } else {
      nc = min(ntc, n - chunk * ntc);
    }
  }
  __device__ void init(long long w0) {
    int lo = 0, hi = nslots - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (woff[mid] <= w0) lo = mid; else hi = mid - 1;
    }
    slot = lo;
    load_slot();
    pos = woff[lo];
    while (slot < nslots) {
      const long long c = stage_cost(nc), chunk_cost = c * spe;
      if (pos + chunk_cost <= w0) { pos += chunk_cost; next_chunk(); continue; }
      const long long kk = (w0 - pos + c - 1) / c;
      if (kk >= spe) { pos += chunk_cost; next_chunk(); }
      else { stage = int(kk); pos += kk * c; }
      break;
    }
  }
  __device__ bool valid(long long w1) const { return slot < nslots && pos < w1; }
  __device__ void advance() { pos += stage_cost(nc); if (++stage == spe) next_chunk(); }
};

__device__ __forceinline__ float round_bf16f(float v) { return __bfloat162float(__float2bfloat16_rn(v)); }

// Stages one row of h (fp32, K values) as int16 in the down pass's operand
// order, with the power-of-two scale of act_shift; returns the row's
// act_inv factor through inv_out (lane 0).
template <int BITS, int LPR, int CPL>
__device__ void stage_h_row(const float* hrow, int16_t* dst, float* inv_out, int lane) {
  using Gm = Geom<BITS, LPR, CPL>;
  constexpr int K = Gm::K;
  float vmax = 0.f;
  for (int hh = lane * 8; hh < K; hh += 256) {
    const float4 a = __ldcg(reinterpret_cast<const float4*>(hrow + hh));
    const float4 b = __ldcg(reinterpret_cast<const float4*>(hrow + hh + 4));
    vmax = fmaxf(vmax, fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(a.z), fabsf(a.w))));
    vmax = fmaxf(vmax, fmaxf(fmaxf(fabsf(b.x), fabsf(b.y)), fmaxf(fabsf(b.z), fabsf(b.w))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
  const int sh = act_shift(vmax);
  const float mul = ldexpf(1.f, sh);
  for (int g0 = lane * Gm::G; g0 < K; g0 += 32 * Gm::G) {
    float v[Gm::G];
#pragma unroll
    for (int q = 0; q < Gm::G / 4; ++q) {
      const float4 u = __ldcg(reinterpret_cast<const float4*>(hrow + g0 + 4 * q));
      v[4 * q] = u.x; v[4 * q + 1] = u.y; v[4 * q + 2] = u.z; v[4 * q + 3] = u.w;
    }
    uint4 parts[Gm::NPART];
    pack_int_order<BITS, Gm::G>(v, mul, parts);
    const int base = staged_offset<BITS, LPR, CPL>(g0);
#pragma unroll
    for (int part = 0; part < Gm::NPART; ++part) *reinterpret_cast<uint4*>(dst + base + part * LPR * 8) = parts[part];
  }
  if (lane == 0) *inv_out = act_inv<BITS>(sh);
}

// Stages the activations of one slot chunk (gate/up: x rows, normalised and
// rounded to bf16 in the stack; down: h rows) as int16 in the operand order.
template <int MODE, int BITS, int LPR, int CPL>
__device__ void stage_chunk(const FusedParams& p, const SRoute& rt, const FCursor& cur, const uint16_t* xsrc,
                            const float* rnorm, const float* h, int16_t* xs, float* tok_inv, float* tok_w,
                            int* tok_pos, int warp, int lane) {
  using Gm = Geom<BITS, LPR, CPL>;
  constexpr int K = Gm::K;
  const bool is_shared = cur.e >= p.cfg.num_experts;
  const int k = p.cfg.top_k, T = p.T;
  const int tbase = cur.chunk * cur.ntc;
  for (int tl = warp; tl < cur.nc; tl += kNCW) {
    const int pos = cur.p0 + tbase + tl;
    if (lane == 0) {
      tok_pos[tl] = pos;
      tok_w[tl] = (MODE == DOWN && !is_shared) ? rt.w[rt.pairs[pos]] : 1.f;
    }
    if (MODE == DOWN) {
      stage_h_row<BITS, LPR, CPL>(h + size_t(pos) * K, xs + size_t(tl) * K, &tok_inv[tl], lane);
      continue;
    }
    const int row = is_shared ? pos - T * k : rt.pairs[pos] / k;
    const float rn = rnorm[row];
    float vmax = 0.f;
    for (int hh = lane * 8; hh < K; hh += 256) {
      const uint4 v = __ldcg(reinterpret_cast<const uint4*>(xsrc + size_t(row) * K + hh));
      const uint32_t q[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int z = 0; z < 4; ++z) {
        vmax = fmaxf(vmax, fabsf(round_bf16f(__uint_as_float(q[z] << 16) * rn)));
        vmax = fmaxf(vmax, fabsf(round_bf16f(__uint_as_float(q[z] & 0xFFFF0000u) * rn)));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
    const int sh = act_shift(vmax);
    const float mul = ldexpf(1.f, sh);
    int16_t* dst = xs + size_t(tl) * K;
    for (int g0 = lane * Gm::G; g0 < K; g0 += 32 * Gm::G) {
      float v[Gm::G];
#pragma unroll
      for (int q = 0; q < Gm::G / 8; ++q) {
        const uint4 u = __ldcg(reinterpret_cast<const uint4*>(xsrc + size_t(row) * K + g0 + 8 * q));
        const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int z = 0; z < 4; ++z) {
          v[8 * q + 2 * z] = round_bf16f(__uint_as_float(wd[z] << 16) * rn);
          v[8 * q + 2 * z + 1] = round_bf16f(__uint_as_float(wd[z] & 0xFFFF0000u) * rn);
        }
      }
      uint4 parts[Gm::NPART];
      pack_int_order<BITS, Gm::G>(v, mul, parts);
      const int base = staged_offset<BITS, LPR, CPL>(g0);
#pragma unroll
      for (int part = 0; part < Gm::NPART; ++part) *reinterpret_cast<uint4*>(dst + base + part * LPR * 8) = parts[part];
    }
    if (lane == 0) tok_inv[tl] = act_inv<BITS>(sh);
  }
}

constexpr int kMaxRE = 8;        // router rows (experts) per CTA

// Stages token t once for the whole layer: one L2 round trip for the row
// (each lane holds whole groups of G elements), RMSNorm factor (stack),
// xhat = bf16(x * r), and the power-of-two scale of act_shift; stored as
// int16 in the gate/up operand order.  Then, from the
// same registers, the token's router logits for the ne <= kMaxRE experts
// whose rows (bf16) are in shared memory at rrows once `rbar` completes
// (rbar == nullptr: they already have): sum_h Wr[e][h] * xhat[h] in fp32
// with exact products, plus the bias.  dst == nullptr skips the int16 row;
// xb_out (if set) receives xhat as bf16 in natural order.
template <int BITS, int LPR, int CPL>
__device__ void stage_token_all(const uint16_t* row, bool stack, int16_t* dst, float* rnorm_out, float* inv_out,
                                uint16_t* xb_out, const uint16_t* rrows, int ne, const float* rbias,
                                float* logit_row, uint64_t* rbar, uint32_t rpar, volatile int* abort_flag,
                                int* status, int lane, unsigned long long* tstamp = nullptr) {
  using Gm = Geom<BITS, LPR, CPL>;
  constexpr int K = Gm::K, G = Gm::G, NG = K / (32 * G);       // groups per lane
  constexpr int NW = G / 8;                                     // 16-byte words per group
  uint4 v[NG][NW];
#pragma unroll
  for (int q = 0; q < NG; ++q)
#pragma unroll
    for (int z = 0; z < NW; ++z)
      v[q][z] = __ldcg(reinterpret_cast<const uint4*>(row + (q * 32 + lane) * G + 8 * z));
  float r = 1.f;
  if (stack) {
    float ss[4] = {0.f, 0.f, 0.f, 0.f};        // four partial sums: short dependency chains
#pragma unroll
    for (int q = 0; q < NG; ++q)
#pragma unroll
      for (int z = 0; z < NW; ++z) {
        const uint32_t w[4] = {v[q][z].x, v[q][z].y, v[q][z].z, v[q][z].w};
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          const float a = __uint_as_float(w[y] << 16), b = __uint_as_float(w[y] & 0xFFFF0000u);
          ss[y] = fmaf(a, a, ss[y]);
          ss[y] = fmaf(b, b, ss[y]);
        }
      }
    float st = (ss[0] + ss[1]) + (ss[2] + ss[3]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) st += __shfl_xor_sync(0xffffffffu, st, o);
    r = 1.0f / sqrtf(st / float(K) + 1e-6f);
    // xhat = bf16(x * r), in place (element 2y in the low half of word y)
#pragma unroll
    for (int q = 0; q < NG; ++q)
#pragma unroll
      for (int z = 0; z < NW; ++z) {
        uint32_t w[4] = {v[q][z].x, v[q][z].y, v[q][z].z, v[q][z].w};
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(w[y] << 16) * r,
                                                          __uint_as_float(w[y] & 0xFFFF0000u) * r);
          w[y] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        v[q][z] = make_uint4(w[0], w[1], w[2], w[3]);
      }
  }
  float vm[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int q = 0; q < NG; ++q)
#pragma unroll
    for (int z = 0; z < NW; ++z) {
      const uint32_t w[4] = {v[q][z].x, v[q][z].y, v[q][z].z, v[q][z].w};
#pragma unroll
      for (int y = 0; y < 4; ++y) {
        vm[y] = fmaxf(vm[y], fabsf(__uint_as_float(w[y] << 16)));
        vm[y] = fmaxf(vm[y], fabsf(__uint_as_float(w[y] & 0xFFFF0000u)));
      }
    }
  float vmax = fmaxf(fmaxf(vm[0], vm[1]), fmaxf(vm[2], vm[3]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
  if (tstamp && lane == 0) tstamp[19] = static_cast<unsigned long long>(clock64());   // the row has arrived
  const int sh = act_shift(vmax);
  const float mul = ldexpf(1.f, sh);
#pragma unroll
  for (int q = 0; q < NG && dst != nullptr; ++q) {
    float vf[G];
#pragma unroll
    for (int z = 0; z < NW; ++z) {
      const uint32_t w[4] = {v[q][z].x, v[q][z].y, v[q][z].z, v[q][z].w};
#pragma unroll
      for (int y = 0; y < 4; ++y) {
        vf[8 * z + 2 * y] = __uint_as_float(w[y] << 16);
        vf[8 * z + 2 * y + 1] = __uint_as_float(w[y] & 0xFFFF0000u);
      }
    }
    uint4 parts[Gm::NPART];
    pack_int_order<BITS, G>(vf, mul, parts);
    const int base = staged_offset<BITS, LPR, CPL>((q * 32 + lane) * G);
#pragma unroll
    for (int part = 0; part < Gm::NPART; ++part) *reinterpret_cast<uint4*>(dst + base + part * LPR * 8) = parts[part];
  }
  if (xb_out != nullptr) {
#pragma unroll
    for (int q = 0; q < NG; ++q)
#pragma unroll
      for (int z = 0; z < NW; ++z) *reinterpret_cast<uint4*>(xb_out + (q * 32 + lane) * G + 8 * z) = v[q][z];
  }
  if (lane == 0) {
    *rnorm_out = r;
    *inv_out = act_inv<BITS>(sh);
  }
  if (tstamp && lane == 0) tstamp[20] = static_cast<unsigned long long>(clock64());   // staged
  if (ne <= 0) return;
  if (rbar != nullptr) {
    if (*abort_flag) return;
    if (!mbar_wait(rbar, rpar, abort_flag)) {
      *abort_flag = 1;
      report_error(status, MOE_ERR_TIMEOUT, 43);
      return;
    }
  }
  // experts in groups of 4 (bounded register use)
#pragma unroll 1
  for (int e0 = 0; e0 < ne; e0 += 4) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int q = 0; q < NG; ++q)
#pragma unroll
      for (int z = 0; z < NW; ++z) {
        const int h0 = (q * 32 + lane) * G + 8 * z;
        const uint32_t xw[4] = {v[q][z].x, v[q][z].y, v[q][z].z, v[q][z].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (e0 + e < ne) {
            const uint4 u = *reinterpret_cast<const uint4*>(rrows + size_t(e0 + e) * K + h0);
            const uint32_t ww[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int y = 0; y < 4; ++y) {
              acc[e] = fmaf(__uint_as_float(ww[y] << 16), __uint_as_float(xw[y] << 16), acc[e]);
              acc[e] = fmaf(__uint_as_float(ww[y] & 0xFFFF0000u), __uint_as_float(xw[y] & 0xFFFF0000u), acc[e]);
            }
          }
        }
      }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (e0 + e < ne) {
        float a = acc[e];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        if (lane == 0) logit_row[e0 + e] = a + (rbias ? rbias[e0 + e] : 0.f);
      }
    }
  }
}

// Router logit of one token and one expert from shared-memory rows (xhat and
// the router row, both bf16 in natural order): fp32 sum of exact products,
// reduced over the warp; lane 0 stores it plus the bias.
template <int K>
__device__ void router_dot(const uint16_t* xrow, const uint16_t* wrow, float bias, float* logit, int lane) {
  float a0 = 0.f, a1 = 0.f;
#pragma unroll
  for (int h = lane * 8; h < K; h += 256) {
    const uint4 xv = *reinterpret_cast<const uint4*>(xrow + h);
    const uint4 wv = *reinterpret_cast<const uint4*>(wrow + h);
    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w}, ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
    for (int y = 0; y < 4; ++y) {
      a0 = fmaf(__uint_as_float(ww[y] << 16), __uint_as_float(xw[y] << 16), a0);
      a1 = fmaf(__uint_as_float(ww[y] & 0xFFFF0000u), __uint_as_float(xw[y] & 0xFFFF0000u), a1);
    }
  }
  float a = a0 + a1;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
  if (lane == 0) *logit = a + bias;
}

// Exclusive scans of two values per consumer thread (all kFCons warps), with
// their totals.  Uses 2 * kFCons ints of shared scratch.
__device__ __forceinline__ int2 block_excl_scan2(int a, int b, int* scratch, int2* total) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int x = a, y = b;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int nx = __shfl_up_sync(0xffffffffu, x, o), ny = __shfl_up_sync(0xffffffffu, y, o);
    if (lane >= o) { x += nx; y += ny; }
  }
  if (lane == 31) { scratch[warp] = x; scratch[kFCons + warp] = y; }
  named_bar_sync(kBarAll, kFCons * 32);
  int bx = 0, by = 0, ax = 0, ay = 0;
#pragma unroll
  for (int w = 0; w < kFCons; ++w) {
    const int sx = scratch[w], sy = scratch[kFCons + w];
    if (w < warp) { bx += sx; by += sy; }
    ax += sx;
    ay += sy;
  }
  named_bar_sync(kBarAll, kFCons * 32);
  *total = make_int2(ax, ay);
  return make_int2(bx + x - a, by + y - b);
}

// Per-group token metadata of the chunk being multiplied.
struct GroupTok {
  float* inv;     // 2^-sh of each staged token
  float* w;       // gate weight (down pass) or 1
  int* pos;       // routed position of each token
  int* xrow;      // pre-staged row of each token (gate/up with every token staged)
};

// Consumer side of one pass over this CTA's stages, for consumer group `grp`
// (warps grp*kNCW ...): walks the same stage sequence as the producer and
// takes the stages whose index has the group's parity.  A group stages the
// tokens of a (slot, chunk) itself when it meets its first stage of it.
// SF = 1: fp8 block scales (one E4M3 byte per block), with the fp32 scales of
// the stage's rows staged after them.
template <int MODE, int BITS, int LPR, int CPL, int PS, int SF>
__device__ void consume_pass(const FusedParams& p, const SRoute& rt, FCursor cur, long long w1, unsigned char* ring,
                             int ring_stride, uint64_t* full, uint64_t* empty, int* consumed, int grp,
                             const uint16_t* xsrc, const float* rnorm, const float* hin, float* out, int out_cols,
                             const int16_t* xs_pre, const float* pre_inv, const float* pre_w, int pre_base,
                             int16_t* xs_grp, const GroupTok& tk, volatile int* abort_flag, int* status,
                             unsigned long long* tacc = nullptr, unsigned long long* tabs = nullptr) {
  using Gm = Geom<BITS, LPR, CPL>;
  constexpr int SSZ = SF ? 1 : 2;                   // bytes per block scale
  constexpr int K = Gm::K;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool timed = tacc != nullptr && threadIdx.x == 0;
  const int wg = warp - grp * kNCW;                 // warp inside the group
  const int gtid = threadIdx.x - grp * kNCW * 32;   // thread inside the group
  const int lg = lane / LPR, lr = lane % LPR;
  const int rl0 = (wg * Gm::RW + lg) * 2;
  // pre: every row already staged in xs_pre -- gate/up: token t at row t,
  // pre_inv[t]; down: routed position q at row q - pre_base with
  // pre_inv / pre_w of that row
  const bool pre = xs_pre != nullptr;
  int staged_slot = -1, staged_chunk = -1;
  bool first_data = true;
  for (; cur.valid(w1); cur.advance()) {
    const int i = (*consumed)++;
    if (i % kFGroups != grp) continue;
    if (cur.slot != staged_slot || cur.chunk != staged_chunk) {
      staged_slot = cur.slot;
      staged_chunk = cur.chunk;
      const unsigned long long ts = timed ? global_ns() : 0;
      named_bar_sync(2 + grp, kNCW * 32);
      if (pre) {
        const int tbase = cur.chunk * cur.ntc;
        const bool is_shared = cur.e >= p.cfg.num_experts;
        for (int tl = gtid; tl < cur.nc; tl += kNCW * 32) {
          const int pos = cur.p0 + tbase + tl;
          const int row = MODE == GATEUP ? (is_shared ? pos - p.T * p.cfg.top_k : rt.pairs[pos] / p.cfg.top_k)
                                         : pos - pre_base;
          tk.pos[tl] = pos;
          tk.xrow[tl] = row;
          tk.inv[tl] = pre_inv[row];
          tk.w[tl] = MODE == GATEUP ? 1.f : pre_w[row];
        }
      } else {
        stage_chunk<MODE, BITS, LPR, CPL>(p, rt, cur, xsrc, rnorm, hin, xs_grp, tk.inv, tk.w, tk.pos, wg, lane);
      }
      named_bar_sync(2 + grp, kNCW * 32);
      if (timed) tacc[1] += global_ns() - ts;
    }
    const int slot = i % kFStages;
    bool ok = !*abort_flag;
    const unsigned long long tw = timed ? global_ns() : 0;
    if (ok && !mbar_wait(&full[slot], (i / kFStages) & 1, abort_flag)) {
      ok = false;
      *abort_flag = 1;
      report_error(status, MOE_ERR_TIMEOUT, 41);
    }
    if (timed) {
      const unsigned long long now = global_ns();
      tacc[0] += now - tw;
      const unsigned long long cyc = static_cast<unsigned long long>(clock64());
      tacc[2] += 1;
      if (tabs && first_data) tabs[0] = cyc;            // first stage's data in
      first_data = false;
    }
    if (ok) {
      const unsigned char* st = ring + slot * ring_stride;
      Rows rows{st + rl0 * Gm::RB, st + Gm::CODE_BYTES + rl0 * (Gm::SPR >> PS) * SSZ, cur.stage * Gm::RPS + rl0,
                code_xor(BITS, p.cfg.half_levels)};
      if (SF) {                                   // the row scales the producer staged after the block scales
        const float* rss = reinterpret_cast<const float*>(st + Gm::CODE_BYTES + Gm::RPS * Gm::SPR);
        rows.rs0 = rss[rl0];
        rows.rs1 = rss[rl0 + 1];
      }
      const int nc = cur.nc;
#pragma unroll 1
      for (int tb = 0; tb < nc; tb += 4) {
        const int nt = min(4, nc - tb);
        const int16_t* xb = pre ? xs_pre : xs_grp + size_t(tb) * K;
        const int* xr = pre ? tk.xrow : nullptr;
        if (nt == 1) rows_dot<MODE, BITS, LPR, CPL, 1, PS, SF>(out, out_cols, rows, xb, tb, lr, tk.inv, tk.w, tk.pos, 1, xr);
        else if (nt == 2) rows_dot<MODE, BITS, LPR, CPL, 2, PS, SF>(out, out_cols, rows, xb, tb, lr, tk.inv, tk.w, tk.pos, 2, xr);
        else rows_dot<MODE, BITS, LPR, CPL, 4, PS, SF>(out, out_cols, rows, xb, tb, lr, tk.inv, tk.w, tk.pos, nt, xr);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
    if (timed && tabs) tabs[1] = static_cast<unsigned long long>(clock64());   // last stage done
  }
}

// Completion publishing of gate/up stages, run by the producer thread: it
// learns that a stage was consumed when it waits for the stage's ring slot
// (the consumers' mbarrier arrivals release their h stores to it), and adds
// the finished stages of each expert slot to gdone[slot] after a gpu-scope
// fence, batched per slot, so no consumer warp stalls on a fence.
// The last slot is flushed as soon as the CTA's last gate/up stage is
// confirmed: holding it until the end would wait on down stages whose
// consumers wait for this very count.
struct Publisher {
  int* gdone;
  int rslot[kFStages];     // expert slot of the stage in each ring slot, -1 = not a gate/up stage
  int acc_slot, acc_cnt;
  int pending;             // gate/up stages issued, not yet confirmed
  bool all_issued;         // the gate/up pass has issued its last stage

  __device__ void reset() {
    for (int r = 0; r < kFStages; ++r) rslot[r] = -1;
    acc_slot = -1;
    acc_cnt = 0;
    pending = 0;
    all_issued = false;
  }
  __device__ void issued_all() {
    all_issued = true;
    if (pending == 0) flush();
  }
  __device__ void flush() {
    if (acc_cnt > 0) {
      __threadfence();
      atomicAdd(&gdone[acc_slot], acc_cnt);
    }
    acc_cnt = 0;
  }
  // the stage that occupied ring slot r has been consumed
  __device__ void consumed(int r) {
    const int u = rslot[r];
    rslot[r] = -1;
    if (u < 0) return;
    if (u != acc_slot) { flush(); acc_slot = u; }
    ++acc_cnt;
    if (--pending == 0 && all_issued) flush();
  }
};

// Producer side of one pass: issues this CTA's stages into the ring.
// SF = 1: the block scales are E4M3 bytes, and the stage's fp32 row scales
// (rs: rows_pe per routed expert; sh_rs: the shared expert) follow them in
// the slot at CODE_BYTES + RPS * SPR.
template <int BITS, int LPR, int CPL, int SF>
__device__ void produce_pass(FCursor cur, long long w1, const uint8_t* codes, const unsigned char* scales,
                             const uint8_t* sh_codes, const unsigned char* sh_scales, size_t expert_code_bytes,
                             size_t expert_scale_count, const float* rs, const float* sh_rs, int rows_pe,
                             unsigned char* ring, int ring_stride, uint64_t* full,
                             uint64_t* empty, int* issued, volatile int* abort_flag, int* status, Publisher& pub,
                             bool gate_up, int block, unsigned long long* tabs = nullptr) {
  using Gm = Geom<BITS, LPR, CPL>;
  // fp8 scales: the E4M3 bytes (RPS * SPR) and the fp32 row scales (RPS * 4)
  // share the slot's scale region, sized for RPS * SPR fp16 scales; the row
  // scales' bulk copy needs a 16-byte aligned destination and size
  static_assert(!SF || (Gm::SPR >= 4 && (Gm::CODE_BYTES + Gm::RPS * Gm::SPR) % 16 == 0 && (Gm::RPS * 4) % 16 == 0),
                "fp8 row scales do not fit the stage's scale region");
  const int first_issue = *issued;
  for (; cur.valid(w1); cur.advance()) {
    const int i = *issued;
    const int slot = i % kFStages;
    if (*abort_flag) return;
    if (i >= kFStages) {
      if (!mbar_wait(&empty[slot], ((i / kFStages) - 1) & 1, abort_flag)) {
        *abort_flag = 1;
        report_error(status, MOE_ERR_TIMEOUT, 42);
        return;
      }
      pub.consumed(slot);
    }
    const bool sh = cur.e >= cur.E;
    const uint8_t* cb = sh ? sh_codes : codes + size_t(cur.e) * expert_code_bytes;
    constexpr int SSZ = SF ? 1 : 2;             // bytes per block scale
    const unsigned char* sb = sh ? sh_scales : scales + size_t(cur.e) * expert_scale_count * SSZ;
    const size_t row0 = size_t(cur.stage) * Gm::RPS;
    unsigned char* dst = ring + slot * ring_stride;
    const int spr = scales_per_row(Gm::K, block);
    const uint32_t sbytes = uint32_t(Gm::RPS) * spr * SSZ;
    constexpr uint32_t RSB = SF ? Gm::RPS * 4 : 0;     // row-scale bytes of the stage
    mbar_arrive_expect_tx(&full[slot], Gm::CODE_BYTES + sbytes + RSB);
    const uint64_t pol = l2_evict_first_policy();
    bulk_g2s_hint(dst, cb + row0 * Gm::RB, Gm::CODE_BYTES, &full[slot], pol);
    bulk_g2s_hint(dst + Gm::CODE_BYTES, sb + row0 * spr * SSZ, sbytes, &full[slot], pol);
    if (SF) {
      const float* rb = sh ? sh_rs : rs + size_t(cur.e) * rows_pe;
      bulk_g2s_hint(dst + Gm::CODE_BYTES + Gm::RPS * Gm::SPR, rb + row0, RSB, &full[slot], pol);
    }
    pub.rslot[slot] = gate_up ? cur.slot : -1;
    if (gate_up) ++pub.pending;
    *issued = i + 1;
    if (tabs) {                                  // first and last issue of the pass
      const unsigned long long now = static_cast<unsigned long long>(clock64());
      if (i == first_issue) tabs[0] = now;
      tabs[1] = now;
    }
  }
}

// After the CTA's last stage is issued: waits (bounded) for the stages still
// in the ring and publishes the gate/up ones.
__device__ void drain_publish(int issued, uint64_t* empty, volatile int* abort_flag, int* status, Publisher& pub) {
  for (int j = max(0, issued - kFStages); j < issued; ++j) {
    const int slot = j % kFStages;
    if (pub.rslot[slot] < 0) continue;
    if (*abort_flag || !mbar_wait(&empty[slot], (j / kFStages) & 1, abort_flag)) {
      if (!*abort_flag) { *abort_flag = 1; report_error(status, MOE_ERR_TIMEOUT, 45); }
      return;
    }
    pub.consumed(slot);
  }
  pub.flush();
}

template <int BITS, int LG, int CG, int LD, int CD, int NPL, int PS, int SF>
__global__ void __launch_bounds__(kFThreads, 1) fused_decode_kernel(const __grid_constant__ FusedParams p) {
  using GU = Geom<BITS, LG, CG>;
  using DN = Geom<BITS, LD, CD>;
  constexpr int RING_STRIDE = GU::STAGE_BYTES > DN::STAGE_BYTES ? GU::STAGE_BYTES : DN::STAGE_BYTES;
  const moe_config& c = p.cfg;
  const int T = p.T, k = c.top_k, E = c.num_experts, H = c.hidden, I = c.inter;
  const int S = c.shared_inter > 0 ? 1 : 0;
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + kFStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kFStages);
  uint64_t* rbar = full + 2 * kFStages + 1;                                // router rows landed
  float* rnorm = reinterpret_cast<float*>(smem + 128);                   // [64]
  float* inv_all = reinterpret_cast<float*>(smem + 384);                 // [64]
  int* snslots = reinterpret_cast<int*>(smem + 640);
  int* scan_scratch = reinterpret_cast<int*>(smem + 768);                // [2 * kFCons]
  int* s_handover = snslots + 1;                                         // 1: tensor-core kernels take the layer
  // [1024, 3072): per-group token metadata, 4 arrays of kMaxNTC each
  float* dinv = reinterpret_cast<float*>(smem + 3072);                   // [64] down rows staged at once
  float* dwt = dinv + kMaxNTC;                                           // [64]
  unsigned char* ring = smem + kFRingOff;
  const int P = T * k;
  int* ri = reinterpret_cast<int*>(smem + p.smem_route_off);
  SRoute rt;
  rt.idx = ri;
  rt.w = reinterpret_cast<float*>(ri + P);
  rt.pairs = ri + 2 * P;
  rt.inv = ri + 3 * P;
  rt.offsets = ri + 4 * P;
  rt.ulist = rt.offsets + (E + 1);
  rt.woff_gu = rt.ulist + (E + 1);
  rt.woff_dn = rt.woff_gu + (E + 2);
  rt.tmask = reinterpret_cast<unsigned*>(rt.woff_dn + (E + 2));
  const int NMW = (T + 31) >> 5;                                          // token mask words per expert
  // tokens: every token (pre-staged) or router chunks in R and G; the two
  // groups' chunk buffers in G (not pre-staged) and D
  int16_t* xs = reinterpret_cast<int16_t*>(smem + p.smem_xs_off);

  char* ws = p.ws;
  int* status = reinterpret_cast<int*>(ws + p.L_.status);
  unsigned* gword = reinterpret_cast<unsigned*>(status + ST_GRID_COUNT);
  float* logits = reinterpret_cast<float*>(ws + p.L_.logits);
  float* hbuf = reinterpret_cast<float*>(ws + p.L_.h);
  float* ybuf = reinterpret_cast<float*>(ws + p.L_.y);
  int* gdone = reinterpret_cast<int*>(ws + p.L_.gdone);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool producer = warp == kFCons;
  const int grp = producer ? 0 : warp / kNCW;
  float* tkb = reinterpret_cast<float*>(smem + 1024 + grp * 4 * kMaxNTC * 4);
  const GroupTok tk{tkb, tkb + kMaxNTC, reinterpret_cast<int*>(tkb + 2 * kMaxNTC),
                    reinterpret_cast<int*>(tkb + 3 * kMaxNTC)};
  int16_t* xs_grp = xs + size_t(grp) * p.grp_xs;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kFStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], kNCW); }
    mbar_init(rbar, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();
  // launched behind the kernel that clears the workspace's status words (a
  // programmatic dependency, so this launch overlaps that one); nothing in
  // the workspace is touched before it has completed
  pdl_wait();
  // the next call's status reset may be scheduled now; it waits for this
  // grid to complete before it clears anything
  pdl_launch_dependents();
  int issued = 0, consumed = 0;
  const unsigned G = gridDim.x;
  const uint16_t* xsrc = p.stack ? p.y : p.x;
  auto all_sync = [&]() { named_bar_sync(kBarAll, kFCons * 32); };
  auto grid_sync = [&]() {
    all_sync();
    if (threadIdx.x == 0 && !*abort_flag && !grid_barrier(gword, G, status)) *abort_flag = 1;
    all_sync();
  };
  // SM clock cycles (fine-grained within the CTA); the layer start and the
  // end of the combine also in %globaltimer ns at [22] / [23], comparable
  // across CTAs
  auto stamp = [&](int l, int i) {
    if (p.timing && l == 0 && threadIdx.x == 0) {
      p.timing[blockIdx.x * kTimePoints + i] = static_cast<unsigned long long>(clock64());
      if (i == 8) p.timing[blockIdx.x * kTimePoints + 22] = global_ns();
      if (i == 7) p.timing[blockIdx.x * kTimePoints + 23] = global_ns();
    }
  };

  for (int l = 0; l < p.L; ++l) {
    const moe_layer_weights& lw = p.w[l];
    stamp(l, 8);
    // ------------------------------------------------------------ phase R
    // (the ring is idle until the routing is done: slot 0 takes this CTA's
    // router rows, slot 3 the top-k scratch)
    const int e0 = int((long long)E * blockIdx.x / G), e1 = int((long long)E * (blockIdx.x + 1) / G);
    if (producer) {
      if (lane == 0) {
        if (e1 > e0) {
          mbar_arrive_expect_tx(rbar, uint32_t(e1 - e0) * H * 2);
          bulk_g2s(ring, lw.router_w + size_t(e0) * H, uint32_t(e1 - e0) * H * 2, rbar);
        }
        if (S) {
          // this CTA's share of the shared expert, into L2 for whoever streams it
          const size_t gu = size_t(2 * I) * H * c.bits / 8, dn = size_t(H) * I * c.bits / 8;
          const size_t a0 = (gu * blockIdx.x / G) & ~size_t(15), a1 = (gu * (blockIdx.x + 1) / G) & ~size_t(15);
          if (a1 > a0) bulk_prefetch_l2(lw.shared_gate_up_codes + a0, uint32_t(a1 - a0));
          const size_t b0 = (dn * blockIdx.x / G) & ~size_t(15), b1 = (dn * (blockIdx.x + 1) / G) & ~size_t(15);
          if (b1 > b0) bulk_prefetch_l2(lw.shared_down_codes + b0, uint32_t(b1 - b0));
        }
      }
    } else {
      // one warp per token: it stages the token (RMSNorm factor in the stack,
      // int16 xhat with its power-of-two scale) -- into the token region, where
      // it stays for gate/up, or, when the tokens do not all fit, into its own
      // row of the idle ring slots 1-2 -- and at once computes the token's
      // router logits for this CTA's experts from their rows in ring slot 0
      for (int e = threadIdx.x; e < NMW * E; e += kFCons * 32) rt.tmask[e] = 0u;
      {
        // this CTA's share of the per-slot gate/up completion counters
        const int z0 = int((long long)(E + 2) * blockIdx.x / G), z1 = int((long long)(E + 2) * (blockIdx.x + 1) / G);
        for (int u = z0 + threadIdx.x; u < z1; u += kFCons * 32) gdone[u] = 0;
      }
      stamp(l, 21);
      // one warp per token: staging and, from the same registers, the
      // token's router logits for this CTA's experts; with fewer tokens than
      // warps, the warps keep xhat (bf16) in the idle ring slots 1-2 instead
      // and then all warps share the (token, expert) dots
      const int ne = e1 - e0;
      const bool few = T < kFCons;
      uint16_t* xb = reinterpret_cast<uint16_t*>(ring + RING_STRIDE);
      bool have_rows = false;
      for (int t = warp; t < T; t += kFCons) {
        stage_token_all<BITS, LG, CG>(xsrc + size_t(t) * H, p.stack != 0, p.pre ? xs + size_t(t) * H : nullptr,
                                      &rnorm[t], &inv_all[t], few ? xb + size_t(t) * H : nullptr,
                                      reinterpret_cast<const uint16_t*>(ring), few ? 0 : ne,
                                      lw.router_bias ? lw.router_bias + e0 : nullptr, logits + size_t(t) * E + e0,
                                      have_rows ? nullptr : rbar, l & 1, abort_flag, status, lane,
                                      (p.timing && l == 0 && t == 0) ? p.timing + blockIdx.x * kTimePoints : nullptr);
        have_rows = !few;
        if (t == 0) stamp(l, 14);
        __syncwarp();
      }
      if (few) {
        all_sync();
        for (int pr = warp; pr < T * ne; pr += kFCons) {
          if (!have_rows) {
            have_rows = true;
            if (*abort_flag) break;
            if (!mbar_wait(rbar, l & 1, abort_flag)) {
              *abort_flag = 1;
              report_error(status, MOE_ERR_TIMEOUT, 43);
              break;
            }
          }
          const int t = pr / ne, e = pr % ne;
          router_dot<GU::K>(xb + size_t(t) * H, reinterpret_cast<const uint16_t*>(ring) + size_t(e) * H,
                            lw.router_bias ? lw.router_bias[e0 + e] : 0.f, logits + size_t(t) * E + e0 + e, lane);
        }
      }
      stamp(l, 15);
      all_sync();
      stamp(l, 0);
      grid_sync();
      stamp(l, 1);
      // ---------------------------------------------------------- phase S
      {
        uint2* tscr = reinterpret_cast<uint2*>(ring + 3 * RING_STRIDE) + warp * 32;
        // CTAs start at different tokens, so their reads of the freshly
        // written logits spread over the L2 lines of all tokens
        for (int tt = warp; tt < T; tt += kFCons) {
          const int t = (tt + int(blockIdx.x)) % T;
          warp_topk<NPL, true>(logits + size_t(t) * E, k, E, rt.idx + t * k, rt.w + t * k, tscr, rt.tmask, t);
        }
      }
      all_sync();
      stamp(l, 9);
      if (P <= 31) {
        // a few pairs (one, two or three tokens): one warp ranks them by
        // (expert, pair id) -- the stable positions -- finds each expert's run,
        // and scans the slots' costs; later phases read offsets[e] and
        // offsets[e + 1] of the picked experts only
        if (warp == 0) {
          const bool act = lane < P;
          const int e = act ? rt.idx[lane] : 0x7FFFFFFF;
          int rank = 0, cnt = 0;
          bool first = act;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int ej = __shfl_sync(0xffffffffu, e, j);
            if (j < P) {
              rank += (ej < e || (ej == e && j < lane)) ? 1 : 0;
              cnt += ej == e ? 1 : 0;
              if (ej == e && j < lane) first = false;
            }
          }
          const unsigned fm = __ballot_sync(0xffffffffu, first);
          int slot = 0;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int ej = __shfl_sync(0xffffffffu, e, j);
            slot += ((fm >> j) & 1u) && ej < e ? 1 : 0;
          }
          if (act) {
            rt.pairs[rank] = lane;
            rt.inv[lane] = rank;
          }
          if (first) {
            rt.ulist[slot] = e;
            rt.offsets[e] = rank;
            rt.offsets[e + 1] = rank + cnt;      // the next picked expert's start, when that is e + 1
          }
          const int U = __popc(fm), ns = U + S;
          if (lane == 0) {
            rt.offsets[E] = P;
            if (S) rt.ulist[U] = E;
            *snslots = ns;
          }
          __syncwarp();
          const PassPlan pg{p.ntc_gu, 2 * I / GU::RPS}, pd{p.ntc_dn, H / DN::RPS};
          int gc = 0, dc = 0;
          if (lane < ns) {
            const int eu = rt.ulist[lane];
            const int n = eu >= E ? T : rt.offsets[eu + 1] - rt.offsets[eu];
            gc = pass_cost(pg, n);
            dc = pass_cost(pd, n);
          }
          int gi = gc, di = dc;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int ng = __shfl_up_sync(0xffffffffu, gi, o), nd = __shfl_up_sync(0xffffffffu, di, o);
            if (lane >= o) { gi += ng; di += nd; }
          }
          if (lane < ns) {
            rt.woff_gu[lane] = gi - gc;
            rt.woff_dn[lane] = di - dc;
          }
          if (lane == 31) {
            rt.woff_gu[ns] = gi;
            rt.woff_dn[ns] = di;
          }
        }
        all_sync();
        stamp(l, 10);
        if (warp == 1 && p.trace && blockIdx.x == 0) {
          for (int q = lane; q < P; q += 32) p.trace[size_t(l) * P + q] = rt.idx[q];
        }
      } else {
        {
          // exclusive scan of the counts and the ascending touched-expert list
          const int EPT = (E + kFCons * 32 - 1) / (kFCons * 32);     // experts per thread
          const int eb = threadIdx.x * EPT;
          int csum = 0, fsum = 0;
          for (int z = 0; z < EPT; ++z) {
            const int e = eb + z;
            int cc = 0;
            if (e < E)
              for (int m = 0; m < NMW; ++m) cc += __popc(rt.tmask[m * E + e]);
            csum += cc;
            fsum += cc > 0 ? 1 : 0;
          }
          int2 tot;
          const int2 run = block_excl_scan2(csum, fsum, scan_scratch, &tot);
          int crun = run.x, frun = run.y;
          for (int z = 0; z < EPT; ++z) {
            const int e = eb + z;
            if (e < E) {
              rt.offsets[e] = crun;
              int cc = 0;
              for (int m = 0; m < NMW; ++m) cc += __popc(rt.tmask[m * E + e]);
              crun += cc;
              if (cc > 0) rt.ulist[frun++] = e;
            }
          }
          if (threadIdx.x == 0) {
            rt.offsets[E] = tot.x;
            if (S) rt.ulist[tot.y] = E;
            *snslots = tot.y + S;
          }
        }
        all_sync();
        stamp(l, 10);
        // stable positions inside each expert's list (pairs in token order): a
        // pair of token t sits after the earlier tokens in its expert's mask, so
        // every CTA derives the same positions, which the passes of different
        // CTAs rely on.  Meanwhile the cost-weighted work prefix of the slots
        // for the two passes.
        for (int q = threadIdx.x; q < P; q += kFCons * 32) {
          const int e = rt.idx[q], t = q / k;
          int r = 0;
          for (int m = 0; m < NMW; ++m) {
            const int tb = t - 32 * m;
            if (tb <= 0) break;
            const unsigned below = tb >= 32 ? 0xFFFFFFFFu : ((1u << tb) - 1u);
            r += __popc(rt.tmask[m * E + e] & below);
          }
          const int pos = rt.offsets[e] + r;
          rt.pairs[pos] = q;
          rt.inv[q] = pos;
        }
        if (warp == 1 && p.trace && blockIdx.x == 0) {
          for (int q = lane; q < P; q += 32) p.trace[size_t(l) * P + q] = rt.idx[q];
        }
        {
          const PassPlan pg{p.ntc_gu, 2 * I / GU::RPS}, pd{p.ntc_dn, H / DN::RPS};
          const int ns = *snslots;
          const int SPT = (ns + kFCons * 32 - 1) / (kFCons * 32);    // slots per thread
          const int u0 = threadIdx.x * SPT;
          int g = 0, d = 0;
          for (int z = 0; z < SPT; ++z) {
            const int u = u0 + z;
            if (u < ns) {
              const int e = rt.ulist[u];
              const int n = e >= E ? T : rt.offsets[e + 1] - rt.offsets[e];
              g += pass_cost(pg, n);
              d += pass_cost(pd, n);
            }
          }
          int2 tot;
          const int2 run = block_excl_scan2(g, d, scan_scratch, &tot);
          int grun = run.x, drun = run.y;
          const int gt = tot.x, dt = tot.y;
          for (int z = 0; z < SPT; ++z) {
            const int u = u0 + z;
            if (u < ns) {
              const int e = rt.ulist[u];
              const int n = e >= E ? T : rt.offsets[e + 1] - rt.offsets[e];
              rt.woff_gu[u] = grun;
              rt.woff_dn[u] = drun;
              grun += pass_cost(pg, n);
              drun += pass_cost(pd, n);
            }
          }
          if (threadIdx.x == 0) { rt.woff_gu[ns] = gt; rt.woff_dn[ns] = dt; }
          if (p.hybrid) {
            // tensor-core work of the same slots: 128-token tiles of each slot
            // over the gate/up (2I/128 row tiles x H/128 k-blocks) and down
            // (H/128 x I/128) matrices
            const int kb_tile = (2 * I / 128) * (H / 128) + (H / 128) * (I / 128);
            int tk = 0;
            for (int z = 0; z < SPT; ++z) {
              const int u = u0 + z;
              if (u < ns) {
                const int e = rt.ulist[u];
                const int n = e >= E ? T : rt.offsets[e + 1] - rt.offsets[e];
                tk += (n + 127) / 128;
              }
            }
            int2 ttot;
            const int2 trun = block_excl_scan2(tk, 0, scan_scratch, &ttot);
            const float per_f = float(gt + dt) / float(G), per_t = float(ttot.x) * kb_tile / float(G);
            const bool tc = p.hybrid == 2 || p.cost_t0 + p.cost_t1 * per_t < p.cost_f0 + p.cost_f1 * per_f;
            if (threadIdx.x == 0) *s_handover = tc ? 1 : 0;
            if (blockIdx.x == 0) {
              if (threadIdx.x == 0) {
                status[ST_COST_F] = gt + dt;
                status[ST_COST_T] = ttot.x * kb_tile;
                status[ST_PATH] = tc ? 1 : 0;
              }
              if (tc) {
                // the routing in the layout the grouped kernels read
                int* g_counts = reinterpret_cast<int*>(ws + p.L_.counts);
                int* g_offsets = reinterpret_cast<int*>(ws + p.L_.offsets);
                int* g_pairs = reinterpret_cast<int*>(ws + p.L_.pairs);
                int* g_inv = reinterpret_cast<int*>(ws + p.L_.inv);
                int* g_ulist = reinterpret_cast<int*>(ws + p.L_.ulist);
                int* g_ntoff = reinterpret_cast<int*>(ws + p.L_.ntoff);
                int* g_idx = reinterpret_cast<int*>(ws + p.L_.topk_idx);
                float* g_w = reinterpret_cast<float*>(ws + p.L_.topk_w);
                for (int e = threadIdx.x; e <= E; e += kFCons * 32) {
                  g_offsets[e] = rt.offsets[e];
                  if (e < E) g_counts[e] = rt.offsets[e + 1] - rt.offsets[e];
                }
                for (int u = threadIdx.x; u < ns; u += kFCons * 32) g_ulist[u] = rt.ulist[u];
                for (int q = threadIdx.x; q < P; q += kFCons * 32) {
                  g_pairs[q] = rt.pairs[q];
                  g_inv[q] = rt.inv[q];
                  g_idx[q] = rt.idx[q];
                  g_w[q] = rt.w[q];
                }
                // token-tile prefix over the slots, in this thread's SPT slots
                int run = trun.x;
                for (int z = 0; z < SPT; ++z) {
                  const int u = u0 + z;
                  if (u < ns) {
                    const int e = rt.ulist[u];
                    const int n = e >= E ? T : rt.offsets[e + 1] - rt.offsets[e];
                    g_ntoff[u] = run;
                    run += (n + 127) / 128;
                  }
                }
                if (threadIdx.x == 0) {
                  g_ntoff[ns] = ttot.x;
                  status[ST_UCOUNT] = ns - S;
                }
              }
            }
          }
        }
      }

    }
    __syncthreads();                 // routing of this layer ready for all warps
    stamp(l, 2);
    if (p.hybrid && *s_handover) break;     // the grouped tensor-core kernels take the layer

    const int ns = *snslots;
    FCursor cg{};
    cg.r = &rt; cg.T = T; cg.k = k; cg.E = E; cg.spe = 2 * I / GU::RPS; cg.ntc = p.ntc_gu;
    cg.woff = rt.woff_gu; cg.nslots = ns;
    const long long tg = rt.woff_gu[ns];
    const long long g0 = tg * blockIdx.x / G, g1 = tg * (blockIdx.x + 1) / G;
    FCursor cd = cg;
    cd.spe = H / DN::RPS; cd.ntc = p.ntc_dn; cd.woff = rt.woff_dn;
    const long long td = rt.woff_dn[ns];
    const long long d0 = td * blockIdx.x / G, d1 = td * (blockIdx.x + 1) / G;

    if (producer) {
      if (lane == 0) {
        Publisher pub;
        pub.gdone = gdone;
        pub.reset();
        if (g0 < g1) {
          cg.init(g0);
          produce_pass<BITS, LG, CG, SF>(cg, g1, lw.gate_up_codes,
                                      reinterpret_cast<const unsigned char*>(lw.gate_up_scales), lw.shared_gate_up_codes,
                                      reinterpret_cast<const unsigned char*>(lw.shared_gate_up_scales),
                                      size_t(2 * I) * H * c.bits / 8,
                                      size_t(2 * I) * (H / c.block), lw.gate_up_row_scales,
                                      lw.shared_gate_up_row_scales, 2 * I, ring, RING_STRIDE, full, empty, &issued,
                                      abort_flag, status, pub, true, c.block,
                                      p.timing && l == 0 ? p.timing + blockIdx.x * kTimePoints + 28 : nullptr);
        }
        pub.issued_all();
        if (d0 < d1) {
          cd.init(d0);
          produce_pass<BITS, LD, CD, SF>(cd, d1, lw.down_codes, reinterpret_cast<const unsigned char*>(lw.down_scales),
                                      lw.shared_down_codes, reinterpret_cast<const unsigned char*>(lw.shared_down_scales),
                                      size_t(H) * I * c.bits / 8, size_t(H) * (I / c.block), lw.down_row_scales,
                                      lw.shared_down_row_scales, H, ring, RING_STRIDE, full, empty, &issued, abort_flag, status, pub, false, c.block,
                                      p.timing && l == 0 ? p.timing + blockIdx.x * kTimePoints + 30 : nullptr);
        }
        drain_publish(issued, empty, abort_flag, status, pub);
      }
    } else {
      // ---------------------------------------------------------- phase G
      if (g0 < g1) {
        cg.init(g0);
        consume_pass<GATEUP, BITS, LG, CG, PS, SF>(p, rt, cg, g1, ring, RING_STRIDE, full, empty, &consumed, grp, xsrc,
                                           rnorm, nullptr, hbuf, I, p.pre ? xs : nullptr, inv_all, nullptr, 0, xs_grp,
                                           tk, abort_flag, status,
                                           p.timing && l == 0 ? p.timing + blockIdx.x * kTimePoints + 11 : nullptr,
                                           p.timing && l == 0 ? p.timing + blockIdx.x * kTimePoints + 24 : nullptr);
      }
      all_sync();
      stamp(l, 3);
      // ---------------------------------------------------------- phase D
      // no grid barrier: the CTA waits only until every slot of its down range
      // has all its gate/up stages published (any CTA may have computed them)
      if (d0 < d1) {
        cd.init(d0);
        // the CTA's stages cover one contiguous range of routed positions:
        // when it fits, all its h rows are staged at once by every warp
        FCursor cw = cd;
        const int lo = cw.p0 + cw.chunk * cw.ntc;
        const int s_first = cw.slot;
        int hi = lo, s_last = cw.slot;
        for (; cw.valid(d1); cw.advance()) {
          hi = max(hi, cw.p0 + cw.chunk * cw.ntc + cw.nc);
          s_last = cw.slot;
        }
        for (int u = s_first + threadIdx.x; u <= s_last; u += kFCons * 32) {
          const int e = rt.ulist[u];
          const int n = e >= E ? T : rt.offsets[e + 1] - rt.offsets[e];
          const unsigned need = unsigned((2 * I / GU::RPS) * ((n + p.ntc_gu - 1) / p.ntc_gu));
          const long long t0 = clock64();
          while (ld_acquire_u32(reinterpret_cast<const unsigned*>(gdone + u)) < need) {
            if (*abort_flag || clock64() - t0 > kWaitLimitCycles) {
              if (!*abort_flag) { *abort_flag = 1; report_error(status, MOE_ERR_TIMEOUT, 44); }
              break;
            }
          }
        }
        all_sync();
        stamp(l, 4);
        const bool dpre = hi - lo <= kMaxNTC && size_t(hi - lo) * DN::K <= p.xs_halves;
        if (dpre) {
          for (int r = warp; r < hi - lo; r += kFCons) {
            const int pos = lo + r;
            stage_h_row<BITS, LD, CD>(hbuf + size_t(pos) * I, xs + size_t(r) * DN::K, &dinv[r], lane);
            if (lane == 0) dwt[r] = pos < P ? rt.w[rt.pairs[pos]] : 1.f;
          }
          all_sync();
        }
        consume_pass<DOWN, BITS, LD, CD, PS, SF>(p, rt, cd, d1, ring, RING_STRIDE, full, empty, &consumed, grp, xsrc,
                                         rnorm, hbuf, ybuf, H, dpre ? xs : nullptr, dinv, dwt, lo, xs_grp, tk,
                                         abort_flag, status,
                                         p.timing && l == 0 ? p.timing + blockIdx.x * kTimePoints + 16 : nullptr,
                                         p.timing && l == 0 ? p.timing + blockIdx.x * kTimePoints + 26 : nullptr);
      }
      all_sync();
      stamp(l, 5);
      grid_sync();
      stamp(l, 6);
      // ---------------------------------------------------------- phase C
      const int units = T * (H / 8);
      const int u0 = int((long long)units * blockIdx.x / G), u1 = int((long long)units * (blockIdx.x + 1) / G);
      for (int u = u0 + threadIdx.x; u < u1; u += kFCons * 32) {
        const int t = u / (H / 8), h0 = (u % (H / 8)) * 8;
        float acc[8];
        if (S) {
          const float* r = ybuf + size_t(P + t) * H + h0;
          const float4 a = __ldcg(reinterpret_cast<const float4*>(r)), b = __ldcg(reinterpret_cast<const float4*>(r + 4));
          acc[0] = a.x; acc[1] = a.y; acc[2] = a.z; acc[3] = a.w; acc[4] = b.x; acc[5] = b.y; acc[6] = b.z; acc[7] = b.w;
        } else {
#pragma unroll
          for (int z = 0; z < 8; ++z) acc[z] = 0.f;
        }
        for (int j = 0; j < k; ++j) {
          const float* r = ybuf + size_t(rt.inv[t * k + j]) * H + h0;
          const float4 a = __ldcg(reinterpret_cast<const float4*>(r)), b = __ldcg(reinterpret_cast<const float4*>(r + 4));
          acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
          acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
        }
        uint16_t* dst = p.y + size_t(t) * H + h0;
        if (p.stack) {
          const uint4 xv = __ldcg(reinterpret_cast<const uint4*>(dst));
          const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
          for (int z = 0; z < 4; ++z) {
            acc[2 * z] += __uint_as_float(xw[z] << 16);
            acc[2 * z + 1] += __uint_as_float(xw[z] & 0xFFFF0000u);
          }
        }
        *reinterpret_cast<uint4*>(dst) = pack_bf16x8(acc);
      }
      stamp(l, 7);
      if (p.stack && l + 1 < p.L) grid_sync();
    }
    __syncthreads();                 // the next layer's routing overwrites this one's
  }
  // the ring is drained: every issued stage was waited on by the consumers
}

template <int BITS, int LG, int CG, int LD, int CD, int NPL, int PS = 0, int SF = 0>
cudaError_t launch_fused_t(const FusedParams& p, int num_sms, cudaStream_t s) {
  using GU = Geom<BITS, LG, CG>;
  using DN = Geom<BITS, LD, CD>;
  FusedParams q = p;
  constexpr int RING_STRIDE = GU::STAGE_BYTES > DN::STAGE_BYTES ? GU::STAGE_BYTES : DN::STAGE_BYTES;
  constexpr int kSmemMax = 227 * 1024;
  const int E = p.cfg.num_experts, T = p.T, k = p.cfg.top_k;
  const int route_bytes = (4 * T * k + 2 * (E + 1) + 2 * (E + 2) + E * ((T + 31) / 32)) * 4;
  if (size_t((E + num_sms - 1) / num_sms) * p.cfg.hidden * 2 > size_t(RING_STRIDE)) return cudaErrorCooperativeLaunchTooLarge;
  if ((E + num_sms - 1) / num_sms > kMaxRE) return cudaErrorCooperativeLaunchTooLarge;
  q.smem_route_off = kFRingOff + kFStages * RING_STRIDE;
  q.smem_xs_off = (q.smem_route_off + route_bytes + 127) & ~127;
  const int avail = kSmemMax - q.smem_xs_off;
  if (avail <= 0) return cudaErrorInvalidValue;
  size_t xs_halves;
  if (size_t(T) * GU::K * 2 <= size_t(avail)) {
    // every token staged once per layer for the router and gate/up
    q.pre = 1;
    q.rtc = T;
    q.ntc_gu = T;
    q.ntc_dn = min(T * (k + 1), min(kMaxNTC, avail / (kFGroups * DN::K * 2)));
    q.grp_xs = q.ntc_dn * DN::K;
    xs_halves = max(size_t(T) * GU::K, size_t(kFGroups) * q.grp_xs);
  } else {
    q.pre = 0;
    q.rtc = avail / (GU::K * 2);
    q.ntc_gu = min(T, min(kMaxNTC, avail / (kFGroups * GU::K * 2)));
    q.ntc_dn = min(T * (k + 1), min(kMaxNTC, avail / (kFGroups * DN::K * 2)));
    q.grp_xs = max(q.ntc_gu * GU::K, q.ntc_dn * DN::K);
    xs_halves = max(size_t(q.rtc) * GU::K, size_t(kFGroups) * q.grp_xs);
  }
  if (q.rtc < 1 || q.ntc_gu < 1 || q.ntc_dn < 1) return cudaErrorInvalidValue;
  // with fewer tokens than consumer warps, xhat rows (bf16) wait in ring slots 1-2
  static_assert(kFCons * 2048 * 2 <= 2 * RING_STRIDE, "xhat rows exceed ring slots 1-2");
  if (T < kFCons && size_t(T) * p.cfg.hidden * 2 > size_t(2) * RING_STRIDE) return cudaErrorCooperativeLaunchTooLarge;
  q.xs_halves = (long long)xs_halves;
  const size_t smem = q.smem_xs_off + xs_halves * 2;
  if (smem > size_t(kSmemMax)) return cudaErrorInvalidValue;
  auto kern = fused_decode_kernel<BITS, LG, CG, LD, CD, NPL, PS, SF>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(num_sms);
  cfg.blockDim = dim3(kFThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  err = cudaLaunchKernelEx(&cfg, kern, q);
  if (err == cudaErrorNotSupported || err == cudaErrorInvalidValue) {
    // no programmatic dependency with a cooperative launch here: launch it
    // plainly (the status words are already cleared by then)
    (void)cudaGetLastError();
    cfg.numAttrs = 1;
    err = cudaLaunchKernelEx(&cfg, kern, q);
  }
  return err;
}

}  // namespace

unsigned long long* g_fused_timing = nullptr;

// Hand-over time models, [0] 4-bit/32, [1] 2-bit/16: layer time in us as
// f0 + f1 * (CUDA-core cost units per CTA) and t0 + t1 * (tensor-core
// k-blocks per CTA), least-squares fits to layer times measured on a B200
// with CUDA graphs (32, 40, 48, 56 and 64 tokens, near-uniform and
// Zipf-skewed routing, 6 layer instances each, both paths: 60 batches per
// format; largest residual 17 us).  On those batches the comparison picks the
// faster path for 57 of 60 (4-bit) and 59 of 60 (2-bit), losing at most
// 2.1 us when it does not.
constexpr float kHyF0[2] = {42.80f, 49.80f}, kHyF1[2] = {0.1381f, 0.1513f};
constexpr float kHyT0[2] = {79.03f, 77.72f}, kHyT1[2] = {0.6034f, 0.6007f};

void set_fused_timing(unsigned long long* buf) { g_fused_timing = buf; }

bool fused_supported(const moe_config& c, int T) {
  if (T < 1 || T > kFMaxTokens || T * c.top_k > kFMaxPairs) return false;
  return c.hidden == 2048 && c.inter == 768 && (c.num_experts % 32) == 0 && c.num_experts <= 1024;
}

int g_decode_path_mode = 0;

void set_decode_path_mode(int mode) { g_decode_path_mode = mode; }
int decode_path_mode() { return g_decode_path_mode; }

cudaError_t launch_fused_decode(const moe_config& c, const moe_layer_weights* layers, int L, const uint16_t* x,
                                uint16_t* y, bool stack, int T, int* trace, char* ws, const Layout& Lw, int num_sms,
                                cudaStream_t s, int hybrid) {
  for (int l0 = 0; l0 < L; l0 += kMaxFusedLayers) {
    FusedParams p{};
    p.cfg = c;
    p.T = T;
    p.L = min(kMaxFusedLayers, L - l0);
    p.stack = stack ? 1 : 0;
    p.x = x;
    p.y = y;
    p.trace = trace ? trace + size_t(l0) * T * c.top_k : nullptr;
    p.timing = l0 == 0 ? g_fused_timing : nullptr;
    p.ws = ws;
    p.L_ = Lw;
    p.hybrid = (hybrid && L == 1) ? hybrid : 0;
    // time models of the layer (us) from per-CTA work: CUDA cores
    // f0 + f1 * cost units, tensor cores t0 + t1 * k-blocks
    if (c.bits == 4) { p.cost_f0 = kHyF0[0]; p.cost_f1 = kHyF1[0]; p.cost_t0 = kHyT0[0]; p.cost_t1 = kHyT1[0]; }
    else { p.cost_f0 = kHyF0[1]; p.cost_f1 = kHyF1[1]; p.cost_t0 = kHyT0[1]; p.cost_t1 = kHyT1[1]; }
    for (int l = 0; l < p.L; ++l) p.w[l] = layers[l0 + l];
    cudaError_t err;
    const int npl = c.num_experts / 32;
    // H = 2048 and I = 768: gate/up 16 lanes x 4 pieces, down 8 lanes x 3 (4-bit)
    //                                  16 lanes x 2 pieces,  4 lanes x 3 (2-bit)
    if (c.bits == 4) {
      switch (npl) {
        case 16: err = c.block == 128 ? launch_fused_t<4, 16, 4, 8, 3, 16, 2>(p, num_sms, s)
                     : c.scale_fmt ? launch_fused_t<4, 16, 4, 8, 3, 16, 0, 1>(p, num_sms, s)
                                   : launch_fused_t<4, 16, 4, 8, 3, 16>(p, num_sms, s); break;
        case 32: err = c.block == 128 ? launch_fused_t<4, 16, 4, 8, 3, 32, 2>(p, num_sms, s)
                     : c.scale_fmt ? launch_fused_t<4, 16, 4, 8, 3, 32, 0, 1>(p, num_sms, s)
                                   : launch_fused_t<4, 16, 4, 8, 3, 32>(p, num_sms, s); break;
        case 8: err = c.block == 128 ? launch_fused_t<4, 16, 4, 8, 3, 8, 2>(p, num_sms, s)
                    : c.scale_fmt ? launch_fused_t<4, 16, 4, 8, 3, 8, 0, 1>(p, num_sms, s)
                                  : launch_fused_t<4, 16, 4, 8, 3, 8>(p, num_sms, s); break;
        default: return cudaErrorInvalidValue;
      }
    } else {
      switch (npl) {
        case 16: err = c.scale_fmt ? launch_fused_t<2, 16, 2, 4, 3, 16, 0, 1>(p, num_sms, s)
                                   : launch_fused_t<2, 16, 2, 4, 3, 16>(p, num_sms, s); break;
        case 32: err = c.scale_fmt ? launch_fused_t<2, 16, 2, 4, 3, 32, 0, 1>(p, num_sms, s)
                                   : launch_fused_t<2, 16, 2, 4, 3, 32>(p, num_sms, s); break;
        case 8: err = c.scale_fmt ? launch_fused_t<2, 16, 2, 4, 3, 8, 0, 1>(p, num_sms, s)
                                  : launch_fused_t<2, 16, 2, 4, 3, 8>(p, num_sms, s); break;
        default: return cudaErrorInvalidValue;
      }
    }
    if (err != cudaSuccess) return err;
  }
  return cudaSuccess;
}

}  // namespace moe
