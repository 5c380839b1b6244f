// Fused decode: a whole MoE layer -- or a stack of layers -- for a small batch
// in one cooperative launch of one CTA per SM.
//
// Same operation as the separate kernels (router logits, top-k with
// renormalised gates, grouping, gate/up + SwiGLU, down, gate-weighted combine
// with the shared expert; in the stack RMSNorm before and the bf16 residual
// after each layer), reorganised so that a decode step pays one launch:
//
//   R  every CTA: RMSNorm factors of the T tokens (stack), router logits of
//      its slice of experts -> global; the producer thread prefetches this
//      CTA's share of the shared expert's bytes into L2          | grid barrier
//   S  every CTA (the same deterministic computation): top-k, gates, stable
//      grouping and the cost-balanced work lists, in shared memory
//   G  gate/up + SwiGLU over the CTA's share of the stages; the producer warp
//      streams them (1-D TMA bulk copies into a 3-deep ring) and runs straight
//      on into the CTA's down-pass stages                        | grid barrier
//   D  down x gate weight -> Y                                   | grid barrier
//   C  combine of the CTA's slice of (token, 8 columns) units    | grid barrier
//                                                                  (stack only)
// Grid barriers: a global counter and generation word; every spin is bounded
// (1 s, then MOE_ERR_TIMEOUT in the status word and the CTA skips the rest).
// Decode is bound by moving expert weights ("125 billion parameters on one
// gaming GPU -- first impressions of Strata + Qwen 3.8 Flash Next", section "In
// brief": compute isn't the blocker); with one launch the HBM stream is not
// interrupted by kernel boundaries.
#include "decode_common.cuh"

namespace moe {

namespace {

using namespace gemv;

constexpr int kFStages = 3;
constexpr int kFMaxTokens = 64;
constexpr int kFMaxPairs = kFMaxTokens * 16;
constexpr int kMaxFusedLayers = 64;
constexpr int kTimePoints = 9;

struct FusedParams {
  moe_config cfg;
  int T, L;
  int stack;                     // 1: x_inout residual stream with RMSNorm; 0: y = layer(x)
  const uint16_t* x;             // layer mode input
  uint16_t* y;                   // layer mode output, or the residual stream (stack)
  int* trace;                    // stack: [L][T][k] selections, or null
  unsigned long long* timing;    // null, or [gridDim][9] %globaltimer stamps of layer 0
  char* ws;
  Layout L_;
  int ntc_gu, ntc_dn;
  int smem_route_off, smem_xs_off, smem_tok_off;
  moe_layer_weights w[kMaxFusedLayers];
};

// ------------------------------------------------------------ grid barrier
// One thread per CTA.  Returns false when the wait gave up.
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ bool grid_barrier(unsigned* count, unsigned* gen, unsigned nblocks, unsigned* passed, int* status) {
  __threadfence();
  const unsigned target = *passed + 1;
  if (atomicAdd(count, 1u) == nblocks - 1) {
    atomicExch(count, 0u);
    __threadfence();
    atomicAdd(gen, 1u);
  } else {
    const unsigned long long t0 = global_ns();
    while (int(ld_acquire_u32(gen) - target) < 0) {
      __nanosleep(64);
      if (global_ns() - t0 > kWaitLimitNs) {
        report_error(status, MOE_ERR_TIMEOUT, 40);
        return false;
      }
    }
  }
  *passed = target;
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
  int* cnt;      // [E] scratch
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

// Stages the activations of one slot chunk (gate/up: x rows, normalised and
// rounded to bf16 in the stack; down: h rows) as fp16 in the decoder's order.
template <int MODE, int BITS, int LPR, int CPL>
__device__ void stage_chunk(const FusedParams& p, const SRoute& rt, const FCursor& cur, const uint16_t* xsrc,
                            const float* rnorm, const float* h, __half* xs, float* tok_inv, float* tok_w,
                            int* tok_pos, int warp, int lane) {
  using Gm = Geom<BITS, LPR, CPL>;
  constexpr int K = Gm::K;
  const bool is_shared = cur.e >= p.cfg.num_experts;
  const int k = p.cfg.top_k, T = p.T;
  const int tbase = cur.chunk * cur.ntc;
  for (int tl = warp; tl < cur.nc; tl += kNCW) {
    const int pos = cur.p0 + tbase + tl;
    const int row = (MODE == GATEUP) ? (is_shared ? pos - T * k : rt.pairs[pos] / k) : pos;
    const float rn = (MODE == GATEUP) ? rnorm[row] : 1.f;
    float vmax = 0.f;
    for (int hh = lane * 8; hh < K; hh += 256) {
      if (MODE == GATEUP) {
        const uint4 v = __ldcg(reinterpret_cast<const uint4*>(xsrc + size_t(row) * K + hh));
        const uint32_t q[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int z = 0; z < 4; ++z) {
          vmax = fmaxf(vmax, fabsf(round_bf16f(__uint_as_float(q[z] << 16) * rn)));
          vmax = fmaxf(vmax, fabsf(round_bf16f(__uint_as_float(q[z] & 0xFFFF0000u) * rn)));
        }
      } else {
        const float* src = h + size_t(row) * K + hh;
        const float4 a = __ldcg(reinterpret_cast<const float4*>(src));
        const float4 b = __ldcg(reinterpret_cast<const float4*>(src + 4));
        vmax = fmaxf(vmax, fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(a.z), fabsf(a.w))));
        vmax = fmaxf(vmax, fmaxf(fmaxf(fabsf(b.x), fabsf(b.y)), fmaxf(fabsf(b.z), fabsf(b.w))));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
    int sh = 0;
    if (vmax > 0.f) {
      int ex;
      frexpf(vmax, &ex);
      sh = min(max(8 - ex, -100), 100);
    }
    const float mul = ldexpf(1.f, sh);
    __half* dst = xs + size_t(tl) * K;
    for (int g0 = lane * Gm::G; g0 < K; g0 += 32 * Gm::G) {
      float v[Gm::G];
      if (MODE == GATEUP) {
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
      } else {
#pragma unroll
        for (int q = 0; q < Gm::G / 4; ++q) {
          const float4 u = __ldcg(reinterpret_cast<const float4*>(h + size_t(row) * K + g0 + 4 * q));
          v[4 * q] = u.x; v[4 * q + 1] = u.y; v[4 * q + 2] = u.z; v[4 * q + 3] = u.w;
        }
      }
      __align__(16) __half hv[Gm::G];
#pragma unroll
      for (int j = 0; j < Gm::G; ++j) hv[decode_slot(BITS, j)] = __float2half_rn(v[j] * mul);
      const int base = staged_offset<BITS, LPR, CPL>(g0);
#pragma unroll
      for (int part = 0; part < Gm::NPART; ++part)
        *reinterpret_cast<uint4*>(dst + base + part * LPR * 8) = *reinterpret_cast<const uint4*>(hv + 8 * part);
    }
    if (lane == 0) {
      tok_inv[tl] = ldexpf(1.f, -sh);
      tok_pos[tl] = pos;
      tok_w[tl] = (MODE == DOWN && !is_shared) ? rt.w[rt.pairs[pos]] : 1.f;
    }
  }
}

// Stages token t once for the whole layer: one L2 round trip for the row
// (each lane holds whole groups of G elements), RMSNorm factor (stack),
// xhat = bf16(x * r), and the power-of-two scale that puts max |xhat| in
// [128, 256); stored as fp16 in the gate/up operand order.
template <int BITS, int LPR, int CPL>
__device__ void stage_token_all(const uint16_t* row, bool stack, __half* dst, float* rnorm_out, float* inv_out,
                                int lane) {
  using Gm = Geom<BITS, LPR, CPL>;
  constexpr int K = Gm::K, G = Gm::G, NG = K / (32 * G);       // groups per lane
  uint4 v[NG][G / 8];
#pragma unroll
  for (int q = 0; q < NG; ++q)
#pragma unroll
    for (int z = 0; z < G / 8; ++z)
      v[q][z] = __ldcg(reinterpret_cast<const uint4*>(row + (q * 32 + lane) * G + 8 * z));
  float r = 1.f;
  if (stack) {
    float ss = 0.f;
#pragma unroll
    for (int q = 0; q < NG; ++q)
#pragma unroll
      for (int z = 0; z < G / 8; ++z) {
        const uint32_t w[4] = {v[q][z].x, v[q][z].y, v[q][z].z, v[q][z].w};
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          const float a = __uint_as_float(w[y] << 16), b = __uint_as_float(w[y] & 0xFFFF0000u);
          ss = fmaf(a, a, ss);
          ss = fmaf(b, b, ss);
        }
      }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    r = 1.0f / sqrtf(ss / float(K) + 1e-6f);
  }
  float vmax = 0.f;
#pragma unroll
  for (int q = 0; q < NG; ++q)
#pragma unroll
    for (int z = 0; z < G / 8; ++z) {
      const uint32_t w[4] = {v[q][z].x, v[q][z].y, v[q][z].z, v[q][z].w};
#pragma unroll
      for (int y = 0; y < 4; ++y) {
        vmax = fmaxf(vmax, fabsf(round_bf16f(__uint_as_float(w[y] << 16) * r)));
        vmax = fmaxf(vmax, fabsf(round_bf16f(__uint_as_float(w[y] & 0xFFFF0000u) * r)));
      }
    }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
  int sh = 0;
  if (vmax > 0.f) {
    int ex;
    frexpf(vmax, &ex);
    sh = min(max(8 - ex, -100), 100);
  }
  const float mul = ldexpf(1.f, sh);
#pragma unroll
  for (int q = 0; q < NG; ++q) {
    __align__(16) __half hv[G];
#pragma unroll
    for (int z = 0; z < G / 8; ++z) {
      const uint32_t w[4] = {v[q][z].x, v[q][z].y, v[q][z].z, v[q][z].w};
#pragma unroll
      for (int y = 0; y < 4; ++y) {
        const int j = 8 * z + 2 * y;
        hv[decode_slot(BITS, j)] = __float2half_rn(round_bf16f(__uint_as_float(w[y] << 16) * r) * mul);
        hv[decode_slot(BITS, j + 1)] = __float2half_rn(round_bf16f(__uint_as_float(w[y] & 0xFFFF0000u) * r) * mul);
      }
    }
    const int base = staged_offset<BITS, LPR, CPL>((q * 32 + lane) * G);
#pragma unroll
    for (int part = 0; part < Gm::NPART; ++part)
      *reinterpret_cast<uint4*>(dst + base + part * LPR * 8) = *reinterpret_cast<const uint4*>(hv + 8 * part);
  }
  if (lane == 0) {
    *rnorm_out = r;
    *inv_out = ldexpf(1.f, -sh);
  }
}

// Router logits of expert e for all T tokens from the staged activations:
// sum_j Wr[e][g0+j] * xs[slot(j)] (exact products), times the token's 2^-sh.
template <int BITS, int LPR, int CPL>
__device__ void router_from_staged(const uint16_t* wrow, float bias, const __half* xs, const float* inv_all, int T,
                                   float* logit_col, int E, int lane) {
  using Gm = Geom<BITS, LPR, CPL>;
  constexpr int K = Gm::K, G = Gm::G, NG = K / (32 * G);
  uint4 wv[NG][G / 8];
#pragma unroll
  for (int q = 0; q < NG; ++q)
#pragma unroll
    for (int z = 0; z < G / 8; ++z) wv[q][z] = ld_stream16(wrow + (q * 32 + lane) * G + 8 * z);
  for (int t = 0; t < T; ++t) {
    const __half* xt = xs + size_t(t) * K;
    float acc = 0.f;
#pragma unroll
    for (int q = 0; q < NG; ++q) {
      const int base = staged_offset<BITS, LPR, CPL>((q * 32 + lane) * G);
      __align__(16) __half xv[G];
#pragma unroll
      for (int part = 0; part < Gm::NPART; ++part)
        *reinterpret_cast<uint4*>(xv + 8 * part) = *reinterpret_cast<const uint4*>(xt + base + part * LPR * 8);
#pragma unroll
      for (int z = 0; z < G / 8; ++z) {
        const uint32_t w[4] = {wv[q][z].x, wv[q][z].y, wv[q][z].z, wv[q][z].w};
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          const int j = 8 * z + 2 * y;
          acc = fmaf(__uint_as_float(w[y] << 16), __half2float(xv[decode_slot(BITS, j)]), acc);
          acc = fmaf(__uint_as_float(w[y] & 0xFFFF0000u), __half2float(xv[decode_slot(BITS, j + 1)]), acc);
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) logit_col[size_t(t) * E] = acc * inv_all[t] + bias;
  }
}

// Exclusive scan of one value per consumer thread (256 threads); also
// returns the total.  Uses 8 ints of shared scratch.
__device__ __forceinline__ int block_excl_scan(int v, int* scratch, int* total) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += n;
  }
  if (lane == 31) scratch[warp] = x;
  named_bar_sync(1, kNCW * 32);
  int before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < kNCW; ++w) {
    const int s = scratch[w];
    if (w < warp) before += s;
    all += s;
  }
  named_bar_sync(1, kNCW * 32);
  *total = all;
  return before + x - v;
}

// Consumer side of one pass over this CTA's stages.
template <int MODE, int BITS, int LPR, int CPL>
__device__ void consume_pass(const FusedParams& p, const SRoute& rt, const moe_layer_weights& lw, FCursor cur,
                             long long w1, unsigned char* ring, int ring_stride, uint64_t* full, uint64_t* empty,
                             int* consumed, const uint16_t* xsrc, const float* rnorm, const float* hin, float* out,
                             int out_cols, __half* xs, float* tok_inv, float* tok_w, int* tok_pos,
                             volatile int* abort_flag, int* status, const float* inv_all = nullptr,
                             int* tok_xrow = nullptr) {
  using Gm = Geom<BITS, LPR, CPL>;
  constexpr int K = Gm::K;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = lane / LPR, lr = lane % LPR;
  const int rl0 = (warp * Gm::RW + grp) * 2;
  const bool pre = inv_all != nullptr;      // every token already staged (gate/up)
  bool first = true;
  for (; cur.valid(w1); cur.advance()) {
    const int i = (*consumed)++;
    if (first || cur.stage == 0) {
      first = false;
      named_bar_sync(1, kNCW * 32);
      if (pre) {
        const int tbase = cur.chunk * cur.ntc;
        const bool is_shared = cur.e >= p.cfg.num_experts;
        for (int tl = threadIdx.x; tl < cur.nc; tl += kNCW * 32) {
          const int pos = cur.p0 + tbase + tl;
          const int tok = is_shared ? pos - p.T * p.cfg.top_k : rt.pairs[pos] / p.cfg.top_k;
          tok_pos[tl] = pos;
          tok_xrow[tl] = tok;
          tok_inv[tl] = inv_all[tok];
          tok_w[tl] = 1.f;
        }
      } else {
        stage_chunk<MODE, BITS, LPR, CPL>(p, rt, cur, xsrc, rnorm, hin, xs, tok_inv, tok_w, tok_pos, warp, lane);
      }
      named_bar_sync(1, kNCW * 32);
    }
    const int slot = i % kFStages;
    bool ok = !*abort_flag;
    if (ok && !mbar_wait(&full[slot], (i / kFStages) & 1, abort_flag)) {
      ok = false;
      *abort_flag = 1;
      report_error(status, MOE_ERR_TIMEOUT, 41);
    }
    if (ok) {
      const unsigned char* st = ring + slot * ring_stride;
      const Rows rows{st + rl0 * Gm::RB, st + Gm::CODE_BYTES + rl0 * Gm::SPR * 2, cur.stage * Gm::RPS + rl0};
      const int nc = cur.nc;
#pragma unroll 1
      for (int tb = 0; tb < nc; tb += 4) {
        const int nt = min(4, nc - tb);
        const __half* xb = pre ? xs : xs + size_t(tb) * K;
        const int* xr = pre ? tok_xrow : nullptr;
        if (nt == 1) rows_dot<MODE, BITS, LPR, CPL, 1>(out, out_cols, rows, xb, tb, lr, tok_inv, tok_w, tok_pos, 1, xr);
        else if (nt == 2) rows_dot<MODE, BITS, LPR, CPL, 2>(out, out_cols, rows, xb, tb, lr, tok_inv, tok_w, tok_pos, 2, xr);
        else rows_dot<MODE, BITS, LPR, CPL, 4>(out, out_cols, rows, xb, tb, lr, tok_inv, tok_w, tok_pos, nt, xr);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
  }
}

// Producer side of one pass: issues this CTA's stages into the ring.
template <int BITS, int LPR, int CPL>
__device__ void produce_pass(FCursor cur, long long w1, const uint8_t* codes, const uint16_t* scales,
                             const uint8_t* sh_codes, const uint16_t* sh_scales, size_t expert_code_bytes,
                             size_t expert_scale_count, unsigned char* ring, int ring_stride, uint64_t* full,
                             uint64_t* empty, int* issued, volatile int* abort_flag, int* status) {
  using Gm = Geom<BITS, LPR, CPL>;
  for (; cur.valid(w1); cur.advance()) {
    const int i = *issued;
    const int slot = i % kFStages;
    if (*abort_flag) return;
    if (i >= kFStages && !mbar_wait(&empty[slot], ((i / kFStages) - 1) & 1, abort_flag)) {
      *abort_flag = 1;
      report_error(status, MOE_ERR_TIMEOUT, 42);
      return;
    }
    const bool sh = cur.e >= cur.E;
    const uint8_t* cb = sh ? sh_codes : codes + size_t(cur.e) * expert_code_bytes;
    const uint16_t* sb = sh ? sh_scales : scales + size_t(cur.e) * expert_scale_count;
    const size_t row0 = size_t(cur.stage) * Gm::RPS;
    unsigned char* dst = ring + slot * ring_stride;
    mbar_arrive_expect_tx(&full[slot], Gm::CODE_BYTES + Gm::SCALE_BYTES);
    bulk_g2s(dst, cb + row0 * Gm::RB, Gm::CODE_BYTES, &full[slot]);
    bulk_g2s(dst + Gm::CODE_BYTES, sb + row0 * Gm::SPR, Gm::SCALE_BYTES, &full[slot]);
    *issued = i + 1;
  }
}

template <int BITS, int LG, int CG, int LD, int CD, int NPL>
__global__ void __launch_bounds__(kThreads, 1) fused_decode_kernel(const __grid_constant__ FusedParams p) {
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
  float* rnorm = reinterpret_cast<float*>(smem + 64);                    // [64]
  int* snslots = reinterpret_cast<int*>(smem + 320);
  float* inv_all = reinterpret_cast<float*>(smem + 384);                 // [64]
  int* tok_xrow = reinterpret_cast<int*>(smem + 640);                    // [64]
  int* scan_scratch = reinterpret_cast<int*>(smem + 896);                // [8]
  unsigned char* ring = smem + 1024;
  int* ri = reinterpret_cast<int*>(smem + p.smem_route_off);
  SRoute rt;
  rt.idx = ri;
  rt.w = reinterpret_cast<float*>(ri + kFMaxPairs);
  rt.pairs = ri + 2 * kFMaxPairs;
  rt.inv = ri + 3 * kFMaxPairs;
  rt.offsets = ri + 4 * kFMaxPairs;
  rt.ulist = rt.offsets + (E + 1);
  rt.woff_gu = rt.ulist + (E + 1);
  rt.woff_dn = rt.woff_gu + (E + 2);
  rt.cnt = rt.woff_dn + (E + 2);
  __half* xs = reinterpret_cast<__half*>(smem + p.smem_xs_off);
  float* tok_inv = reinterpret_cast<float*>(smem + p.smem_tok_off);
  float* tok_w = tok_inv + kMaxNTC;
  int* tok_pos = reinterpret_cast<int*>(tok_w + kMaxNTC);

  char* ws = p.ws;
  int* status = reinterpret_cast<int*>(ws + p.L_.status);
  unsigned* gcount = reinterpret_cast<unsigned*>(status + ST_GRID_COUNT);
  unsigned* ggen = reinterpret_cast<unsigned*>(status + ST_GRID_GEN);
  float* logits = reinterpret_cast<float*>(ws + p.L_.logits);
  float* hbuf = reinterpret_cast<float*>(ws + p.L_.h);
  float* ybuf = reinterpret_cast<float*>(ws + p.L_.y);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool producer = warp == kNCW;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kFStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], kNCW); }
    *abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();
  unsigned passed = 0;                 // grid barriers passed (thread 0 only)
  int issued = 0, consumed = 0;
  const unsigned G = gridDim.x;
  const uint16_t* xsrc = p.stack ? p.y : p.x;

  for (int l = 0; l < p.L; ++l) {
    const moe_layer_weights& lw = p.w[l];
    if (p.timing && l == 0 && threadIdx.x == 0) p.timing[blockIdx.x * kTimePoints + 8] = global_ns();
    // ------------------------------------------------------------ phase R
    if (producer) {
      if (lane == 0 && S) {
        // this CTA's share of the shared expert, into L2 for whoever streams it
        const size_t gu = size_t(2 * I) * H * c.bits / 8, dn = size_t(H) * I * c.bits / 8;
        const size_t a0 = (gu * blockIdx.x / G) & ~size_t(15), a1 = (gu * (blockIdx.x + 1) / G) & ~size_t(15);
        if (a1 > a0) bulk_prefetch_l2(lw.shared_gate_up_codes + a0, uint32_t(a1 - a0));
        const size_t b0 = (dn * blockIdx.x / G) & ~size_t(15), b1 = (dn * (blockIdx.x + 1) / G) & ~size_t(15);
        if (b1 > b0) bulk_prefetch_l2(lw.shared_down_codes + b0, uint32_t(b1 - b0));
      }
    } else {
      // tokens: RMSNorm factors (stack), identical in every CTA; when all T
      // fit, each token is staged once here for the router and gate/up
      const bool xall = p.ntc_gu >= T;
      if (xall) {
        for (int t = warp; t < T; t += kNCW)
          stage_token_all<BITS, LG, CG>(xsrc + size_t(t) * H, p.stack != 0, xs + size_t(t) * H, &rnorm[t],
                                        &inv_all[t], lane);
      } else {
        for (int t = warp; t < T; t += kNCW) {
          float ss = 0.f;
          if (p.stack) {
            for (int hh = lane * 8; hh < H; hh += 256) {
              const uint4 v = __ldcg(reinterpret_cast<const uint4*>(xsrc + size_t(t) * H + hh));
              const uint32_t q[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int z = 0; z < 4; ++z) {
                const float a = __uint_as_float(q[z] << 16), b = __uint_as_float(q[z] & 0xFFFF0000u);
                ss = fmaf(a, a, ss);
                ss = fmaf(b, b, ss);
              }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
          }
          if (lane == 0) rnorm[t] = p.stack ? 1.0f / sqrtf(ss / float(H) + 1e-6f) : 1.f;
        }
      }
      named_bar_sync(1, kNCW * 32);
      // router logits of this CTA's experts: one warp per expert row
      const int e0 = int((long long)E * blockIdx.x / G), e1 = int((long long)E * (blockIdx.x + 1) / G);
      for (int e = e0 + warp; e < e1; e += kNCW) {
        const uint16_t* wr = lw.router_w + size_t(e) * H;
        const float b = lw.router_bias ? lw.router_bias[e] : 0.f;
        if (xall) {
          router_from_staged<BITS, LG, CG>(wr, b, xs, inv_all, T, logits + e, E, lane);
          continue;
        }
        constexpr int RPL = 2048 / 256;      // 16-byte pieces of the row per lane (H = 2048)
        uint4 wv[RPL];
#pragma unroll
        for (int q = 0; q < RPL; ++q) wv[q] = ld_stream16(wr + (q * 32 + lane) * 8);
        for (int t = 0; t < T; ++t) {
          const float rn = rnorm[t];
          float acc = 0.f;
#pragma unroll
          for (int q = 0; q < RPL; ++q) {
            const uint4 xv = __ldcg(reinterpret_cast<const uint4*>(xsrc + size_t(t) * H + (q * 32 + lane) * 8));
            const uint32_t wa[4] = {wv[q].x, wv[q].y, wv[q].z, wv[q].w};
            const uint32_t xa[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
            for (int z = 0; z < 4; ++z) {
              acc = fmaf(__uint_as_float(wa[z] << 16), round_bf16f(__uint_as_float(xa[z] << 16) * rn), acc);
              acc = fmaf(__uint_as_float(wa[z] & 0xFFFF0000u), round_bf16f(__uint_as_float(xa[z] & 0xFFFF0000u) * rn), acc);
            }
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
          if (lane == 0) logits[size_t(t) * E + e] = acc + b;
        }
      }
      named_bar_sync(1, kNCW * 32);
      if (p.timing && l == 0 && threadIdx.x == 0) p.timing[blockIdx.x * kTimePoints + 0] = global_ns();
      if (threadIdx.x == 0 && !*abort_flag && !grid_barrier(gcount, ggen, G, &passed, status)) *abort_flag = 1;
      named_bar_sync(1, kNCW * 32);
      if (p.timing && l == 0 && threadIdx.x == 0) p.timing[blockIdx.x * kTimePoints + 1] = global_ns();
      // ---------------------------------------------------------- phase S
      for (int e = threadIdx.x; e < E; e += kNCW * 32) rt.cnt[e] = 0;
      for (int t = warp; t < T; t += kNCW) warp_topk_fast<NPL, true>(logits + size_t(t) * E, k, E, rt.idx + t * k, rt.w + t * k);
      named_bar_sync(1, kNCW * 32);
      for (int q = threadIdx.x; q < T * k; q += kNCW * 32) atomicAdd(&rt.cnt[rt.idx[q]], 1);
      named_bar_sync(1, kNCW * 32);
      {
        // exclusive scan of the counts and the ascending touched-expert list;
        // cnt becomes each expert's fill cursor
        const int EPT = (E + kNCW * 32 - 1) / (kNCW * 32);      // experts per thread (<= 4)
        const int eb = threadIdx.x * EPT;
        int csum = 0, fsum = 0;
        for (int z = 0; z < EPT; ++z) {
          const int e = eb + z;
          const int cc = e < E ? rt.cnt[e] : 0;
          csum += cc;
          fsum += cc > 0 ? 1 : 0;
        }
        int ctot, ftot;
        int crun = block_excl_scan(csum, scan_scratch, &ctot);
        int frun = block_excl_scan(fsum, scan_scratch, &ftot);
        for (int z = 0; z < EPT; ++z) {
          const int e = eb + z;
          if (e < E) {
            const int cc = rt.cnt[e];
            rt.offsets[e] = crun;
            rt.cnt[e] = crun;
            crun += cc;
            if (cc > 0) rt.ulist[frun++] = e;
          }
        }
        if (threadIdx.x == 0) {
          rt.offsets[E] = ctot;
          if (S) rt.ulist[ftot] = E;
          *snslots = ftot + S;
        }
      }
      named_bar_sync(1, kNCW * 32);
      // stable positions inside each expert's list (pairs in token order), by
      // warp 0 over 32 pairs at a time: every CTA derives the same positions,
      // which the passes of different CTAs rely on.  Meanwhile the
      // cost-weighted work prefix of the slots for the two passes.
      if (warp == 0) {
        for (int base = 0; base < T * k; base += 32) {
          const int q = base + lane;
          const int e = q < T * k ? rt.idx[q] : -1 - lane;
          const unsigned same = __match_any_sync(0xffffffffu, e);
          const int rank = __popc(same & ((1u << lane) - 1u));
          const int start = q < T * k ? rt.cnt[e] : 0;
          __syncwarp();
          if (q < T * k) {
            const int pos = start + rank;
            rt.pairs[pos] = q;
            rt.inv[q] = pos;
            if ((same >> lane) == 1u) rt.cnt[e] = start + rank + 1;     // last of its expert in this group
          }
          __syncwarp();
        }
      } else if (warp == 1 && p.trace && blockIdx.x == 0) {
        for (int q = lane; q < T * k; q += 32) p.trace[size_t(l) * T * k + q] = rt.idx[q];
      }
      {
        const PassPlan pg{p.ntc_gu, 2 * I / GU::RPS}, pd{p.ntc_dn, H / DN::RPS};
        const int ns = *snslots;
        const int SPT = (ns + kNCW * 32 - 1) / (kNCW * 32);     // slots per thread
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
        int gt, dt;
        int grun = block_excl_scan(g, scan_scratch, &gt);
        int drun = block_excl_scan(d, scan_scratch, &dt);
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
      }
    }
    __syncthreads();                 // routing of this layer ready for all warps
    if (p.timing && l == 0 && threadIdx.x == 0) p.timing[blockIdx.x * kTimePoints + 2] = global_ns();

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
        if (g0 < g1) {
          cg.init(g0);
          produce_pass<BITS, LG, CG>(cg, g1, lw.gate_up_codes, lw.gate_up_scales, lw.shared_gate_up_codes,
                                      lw.shared_gate_up_scales, size_t(2 * I) * H * c.bits / 8,
                                      size_t(2 * I) * (H / c.block), ring, RING_STRIDE, full, empty, &issued,
                                      abort_flag, status);
        }
        if (d0 < d1) {
          cd.init(d0);
          produce_pass<BITS, LD, CD>(cd, d1, lw.down_codes, lw.down_scales, lw.shared_down_codes,
                                      lw.shared_down_scales, size_t(H) * I * c.bits / 8, size_t(H) * (I / c.block),
                                      ring, RING_STRIDE, full, empty, &issued, abort_flag, status);
        }
      }
    } else {
      // ---------------------------------------------------------- phase G
      if (g0 < g1) {
        cg.init(g0);
        const bool xall = p.ntc_gu >= T;
        consume_pass<GATEUP, BITS, LG, CG>(p, rt, lw, cg, g1, ring, RING_STRIDE, full, empty, &consumed, xsrc,
                                           rnorm, nullptr, hbuf, I, xs, tok_inv, tok_w, tok_pos, abort_flag, status,
                                           xall ? inv_all : nullptr, tok_xrow);
      }
      named_bar_sync(1, kNCW * 32);
      if (p.timing && l == 0 && threadIdx.x == 0) p.timing[blockIdx.x * kTimePoints + 3] = global_ns();
      if (threadIdx.x == 0 && !*abort_flag && !grid_barrier(gcount, ggen, G, &passed, status)) *abort_flag = 1;
      named_bar_sync(1, kNCW * 32);
      if (p.timing && l == 0 && threadIdx.x == 0) p.timing[blockIdx.x * kTimePoints + 4] = global_ns();
      // ---------------------------------------------------------- phase D
      if (d0 < d1) {
        cd.init(d0);
        consume_pass<DOWN, BITS, LD, CD>(p, rt, lw, cd, d1, ring, RING_STRIDE, full, empty, &consumed, xsrc,
                                         rnorm, hbuf, ybuf, H, xs, tok_inv, tok_w, tok_pos, abort_flag, status);
      }
      named_bar_sync(1, kNCW * 32);
      if (p.timing && l == 0 && threadIdx.x == 0) p.timing[blockIdx.x * kTimePoints + 5] = global_ns();
      if (threadIdx.x == 0 && !*abort_flag && !grid_barrier(gcount, ggen, G, &passed, status)) *abort_flag = 1;
      named_bar_sync(1, kNCW * 32);
      if (p.timing && l == 0 && threadIdx.x == 0) p.timing[blockIdx.x * kTimePoints + 6] = global_ns();
      // ---------------------------------------------------------- phase C
      const int units = T * (H / 8);
      const int u0 = int((long long)units * blockIdx.x / G), u1 = int((long long)units * (blockIdx.x + 1) / G);
      for (int u = u0 + threadIdx.x; u < u1; u += kNCW * 32) {
        const int t = u / (H / 8), h0 = (u % (H / 8)) * 8;
        float acc[8];
        if (S) {
          const float* r = ybuf + size_t(T * k + t) * H + h0;
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
        __align__(16) uint16_t ob[8];
#pragma unroll
        for (int z = 0; z < 8; ++z) ob[z] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[z]));
        *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(ob);
      }
      if (p.timing && l == 0 && threadIdx.x == 0) p.timing[blockIdx.x * kTimePoints + 7] = global_ns();
      if (p.stack && l + 1 < p.L) {
        named_bar_sync(1, kNCW * 32);
        if (threadIdx.x == 0 && !*abort_flag && !grid_barrier(gcount, ggen, G, &passed, status)) *abort_flag = 1;
        named_bar_sync(1, kNCW * 32);
      }
    }
    __syncthreads();                 // the next layer's routing overwrites this one's
  }
  // the ring is drained: every issued stage was waited on by the consumers
}

template <int BITS, int LG, int CG, int LD, int CD, int NPL>
cudaError_t launch_fused_t(const FusedParams& p, int num_sms, cudaStream_t s) {
  using GU = Geom<BITS, LG, CG>;
  using DN = Geom<BITS, LD, CD>;
  FusedParams q = p;
  constexpr int RING_STRIDE = GU::STAGE_BYTES > DN::STAGE_BYTES ? GU::STAGE_BYTES : DN::STAGE_BYTES;
  const int E = p.cfg.num_experts;
  const int route_bytes = (4 * kFMaxPairs + 2 * (E + 1) + 2 * (E + 2) + E) * 4;
  q.smem_route_off = 1024 + kFStages * RING_STRIDE;
  q.smem_tok_off = q.smem_route_off + ((route_bytes + 127) & ~127);
  q.smem_xs_off = q.smem_tok_off + kMaxNTC * 12 + 128;
  q.smem_xs_off = (q.smem_xs_off + 127) & ~127;
  const int avail = 227 * 1024 - q.smem_xs_off - 256;
  q.ntc_gu = min(p.T, min(kMaxNTC, (avail / (GU::K * 2)) & ~1));
  q.ntc_dn = min(p.T * (p.cfg.top_k + 1), min(kMaxNTC, (avail / (DN::K * 2)) & ~1));
  if (q.ntc_gu < 1 || q.ntc_dn < 1) return cudaErrorInvalidValue;
  const size_t smem = q.smem_xs_off + size_t(max(q.ntc_gu * GU::K, q.ntc_dn * DN::K)) * 2;
  auto kern = fused_decode_kernel<BITS, LG, CG, LD, CD, NPL>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(num_sms);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, q);
}

}  // namespace

unsigned long long* g_fused_timing = nullptr;

void set_fused_timing(unsigned long long* buf) { g_fused_timing = buf; }

bool fused_supported(const moe_config& c, int T) {
  if (T < 1 || T > kFMaxTokens || T * c.top_k > kFMaxPairs) return false;
  return c.hidden == 2048 && c.inter == 768 && (c.num_experts % 32) == 0 && c.num_experts <= 1024;
}

cudaError_t launch_fused_decode(const moe_config& c, const moe_layer_weights* layers, int L, const uint16_t* x,
                                uint16_t* y, bool stack, int T, int* trace, char* ws, const Layout& Lw, int num_sms,
                                cudaStream_t s) {
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
    for (int l = 0; l < p.L; ++l) p.w[l] = layers[l0 + l];
    cudaError_t err;
    const int npl = c.num_experts / 32;
    // H = 2048 and I = 768: gate/up 16 lanes x 4 pieces, down 8 lanes x 3 (4-bit)
    //                                  32 lanes x 1 piece,   4 lanes x 3 (2-bit)
    if (c.bits == 4) {
      switch (npl) {
        case 16: err = launch_fused_t<4, 16, 4, 8, 3, 16>(p, num_sms, s); break;
        case 32: err = launch_fused_t<4, 16, 4, 8, 3, 32>(p, num_sms, s); break;
        case 8: err = launch_fused_t<4, 16, 4, 8, 3, 8>(p, num_sms, s); break;
        default: return cudaErrorInvalidValue;
      }
    } else {
      switch (npl) {
        case 16: err = launch_fused_t<2, 32, 1, 4, 3, 16>(p, num_sms, s); break;
        case 32: err = launch_fused_t<2, 32, 1, 4, 3, 32>(p, num_sms, s); break;
        case 8: err = launch_fused_t<2, 32, 1, 4, 3, 8>(p, num_sms, s); break;
        default: return cudaErrorInvalidValue;
      }
    }
    if (err != cudaSuccess) return err;
  }
  return cudaSuccess;
}

}  // namespace moe
