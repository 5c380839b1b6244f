// Decode path: grouped GEMV over the packed rows of the selected experts.
//
// Per selected expert e with token list L_e (and the shared expert with all T
// tokens): gate/up pass h = silu(W_gate x) * (W_up x), down pass
// Y = w_(t,e) * W_down h.  The expert FFN replaces the dense FFN
// ("Running a 125B Model on a Single RTX 5090: Strata Benchmarks Qwen3.8 Flash
// Next", section "Layer 1: On-Demand MoE Expert Scheduling"); decode is bound
// by moving expert weights, not by arithmetic ("125 billion parameters on one
// gaming GPU -- first impressions of Strata + Qwen 3.8 Flash Next", section "In
// brief": compute isn't the blocker).
//
// Design: every CTA takes an equal contiguous share of all (expert, row-group)
// work units, so HBM bytes are balanced across SMs.  A producer warp streams
// each stage's packed rows and scales into a shared-memory ring with 1-D bulk
// copies; the consumer warps turn each code field into a signed byte (16 q or
// 64 q), multiply with the activations staged in shared memory as int16
// (scaled per token by a power of two) with dp2a, sum each block exactly in
// int32 and the blocks in fp32 with the block's scale, then reduce across the
// lanes of the row with shuffles.  No atomics: every output element is written
// once.  This kernel also serves every shape and layer the single-launch
// decode kernel leaves out (other hidden/intermediate sizes, the gated shared
// expert) and, at every batch size, layers with fp8 (E4M3) block scales, which
// the tensor-core prefill does not read.
#include "decode_common.cuh"

namespace moe {

namespace {

using namespace gemv;

struct FfnArgs {
  const uint8_t* codes;          // routed pool
  const unsigned char* scales;   // fp16 or (sf = 1) E4M3 block scales
  const uint8_t* sh_codes;       // shared expert (or null)
  const unsigned char* sh_scales;
  const float* row_scales;       // sf = 1: fp32 scale per row of each routed expert
  const float* sh_row_scales;    // sf = 1: of the shared expert
  int sf;                        // scale format: 0 fp16, 1 E4M3 + row scale
  size_t expert_code_bytes;      // per routed expert
  size_t expert_scale_count;
  int rows;                      // rows per expert (2I gate/up, H down)
  int block;                     // elements per scale
  uint32_t xk;                   // code_xor of the format
  int out_cols;                  // columns of the output buffer (I gate/up, H down)
  int ntc;                       // tokens staged per chunk
  const uint16_t* xin;           // GATEUP: [T][K] bf16 activations
  const float* hin;              // DOWN:   [P][K] fp32 intermediate
  float* out;                    // GATEUP: h [P][I]; DOWN: Y [P][H]
  int* status;
  RouteView rv;
};

// Walks the stages (slot, token chunk, row stage) whose start lies in this
// CTA's share [w0, w1) of the pass's cost (see stage_cost); producer and
// consumers walk the same sequence.
struct Cursor {
  const RouteView* rv;
  int nslots, spe, ntc;
  int slot, n, p0, e, chunk, nc, stage;
  long long pos;               // cost position of the current stage's start

  __device__ void load_slot() {
    slot_range(*rv, slot, &e, &p0, &n);
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
      if (__ldcg(rv->woff + mid) <= w0) lo = mid; else hi = mid - 1;
    }
    slot = lo;
    load_slot();
    pos = __ldcg(rv->woff + lo);
    while (slot < nslots) {
      const long long c = stage_cost(nc), chunk_cost = c * spe;
      if (pos + chunk_cost <= w0) {
        pos += chunk_cost;
        next_chunk();
        continue;
      }
      const long long k = (w0 - pos + c - 1) / c;     // first stage starting at or after w0
      if (k >= spe) {
        pos += chunk_cost;
        next_chunk();
      } else {
        stage = int(k);
        pos += k * c;
      }
      break;
    }
  }
  __device__ bool valid(long long w1) const { return slot < nslots && pos < w1; }
  __device__ void advance() {
    pos += stage_cost(nc);
    if (++stage == spe) next_chunk();
  }
};

template <int MODE, int BITS, int LPR, int CPL, int PS, int SF>
__global__ void __launch_bounds__(kThreads, 1) ffn_tma_kernel(FfnArgs a) {
  constexpr int SSZ = SF ? 1 : 2;               // bytes per block scale
  using Gm = Geom<BITS, LPR, CPL>;
  constexpr int K = Gm::K;
  constexpr int NTB = 4;                        // tokens per register block
  const int ntc = a.ntc;
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kStages);
  unsigned char* ring = smem + 256;
  int16_t* xs = reinterpret_cast<int16_t*>(ring + kStages * Gm::STAGE_BYTES);     // [ntc][K]
  float* tok_inv = reinterpret_cast<float*>(xs + size_t(ntc) * K);
  float* tok_w = tok_inv + kMaxNTC;
  int* tok_pos = reinterpret_cast<int*>(tok_w + kMaxNTC);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool producer = warp == kNCW;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kNCW);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();

  // The weights never depend on the previous kernel; routing was final before
  // that kernel started.  Only the activations (h in the down pass) do.
  if (MODE == GATEUP || !producer) pdl_wait();
  pdl_launch_dependents();

  const RouteView& rv = a.rv;
  const int nslots = __ldcg(rv.status + ST_UCOUNT) + rv.shared;
  const long long total = __ldcg(rv.woff + nslots);
  const long long w0 = total * blockIdx.x / gridDim.x;
  const long long w1 = total * (blockIdx.x + 1) / gridDim.x;
  if (w0 >= w1) return;
  Cursor cur;
  cur.rv = &rv;
  cur.nslots = nslots;
  cur.spe = a.rows / Gm::RPS;
  cur.ntc = ntc;
  cur.init(w0);

  if (producer) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0;
      for (; cur.valid(w1); cur.advance()) {
        const int slot = issued % kStages;
        if (*abort_flag) break;
        if (issued >= kStages && !mbar_wait(&empty[slot], ((issued / kStages) - 1) & 1, abort_flag)) {
          *abort_flag = 1;
          report_error(a.status, MOE_ERR_TIMEOUT, 1);
          break;
        }
        const bool sh = cur.e >= rv.E;
        const uint8_t* cb = sh ? a.sh_codes : a.codes + size_t(cur.e) * a.expert_code_bytes;
        const unsigned char* sb = sh ? a.sh_scales : a.scales + size_t(cur.e) * a.expert_scale_count * SSZ;
        const size_t row0 = size_t(cur.stage) * Gm::RPS;
        unsigned char* dst = ring + slot * Gm::STAGE_BYTES;
        const int spr = scales_per_row(Gm::K, a.block);
        const uint32_t sbytes = uint32_t(Gm::RPS) * spr * SSZ;
        mbar_arrive_expect_tx(&full[slot], Gm::CODE_BYTES + sbytes);
        const uint64_t pol = l2_evict_first_policy();      // weight bytes are read once
        bulk_g2s_hint(dst, cb + row0 * Gm::RB, Gm::CODE_BYTES, &full[slot], pol);
        bulk_g2s_hint(dst + Gm::CODE_BYTES, sb + row0 * spr * SSZ, sbytes, &full[slot], pol);
        ++issued;
      }
      // never leave with copies in flight
      for (int i = max(0, issued - kStages); i < issued; ++i)
        if (!mbar_wait(&full[i % kStages], (i / kStages) & 1, nullptr)) report_error(a.status, MOE_ERR_TIMEOUT, 2);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int grp = lane / LPR, lr = lane % LPR;
  const int rl0 = (warp * Gm::RW + grp) * 2;     // local rows rl0, rl0+1 of each stage
  bool first = true;
  for (int i = 0; cur.valid(w1); ++i, cur.advance()) {
    const int nc = cur.nc;
    if (first || cur.stage == 0) {
      first = false;
      // (re)stage the activations of this slot's token chunk
      const bool is_shared = cur.e >= rv.E;
      const int tbase = cur.chunk * ntc;
      named_bar_sync(1, kNCW * 32);
      for (int tl = warp; tl < nc; tl += kNCW) {
        const int p = cur.p0 + tbase + tl;
        const int row = (MODE == GATEUP) ? (is_shared ? p - rv.T * rv.k : __ldcg(rv.pairs + p) / rv.k) : p;
        float vmax = 0.f;
        if (MODE == GATEUP) {
          const uint16_t* src = a.xin + size_t(row) * K;
          for (int h = lane * 8; h < K; h += 256) {
            const uint4 v = __ldcg(reinterpret_cast<const uint4*>(src + h));
            const uint32_t q[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int z = 0; z < 4; ++z) {
              vmax = fmaxf(vmax, fabsf(__uint_as_float(q[z] << 16)));
              vmax = fmaxf(vmax, fabsf(__uint_as_float(q[z] & 0xFFFF0000u)));
            }
          }
        } else {
          const float* src = a.hin + size_t(row) * K;
          for (int h = lane * 4; h < K; h += 128) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(src + h));
            vmax = fmaxf(vmax, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
        const int sh = act_shift(vmax);
        const float mul = ldexpf(1.f, sh);
        int16_t* dst = xs + size_t(tl) * K;
        for (int g0 = lane * Gm::G; g0 < K; g0 += 32 * Gm::G) {
          float v[Gm::G];
          if (MODE == GATEUP) {
            const uint16_t* src = a.xin + size_t(row) * K + g0;
#pragma unroll
            for (int q = 0; q < Gm::G / 8; ++q) {
              const uint4 u = __ldcg(reinterpret_cast<const uint4*>(src + 8 * q));
              const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
              for (int z = 0; z < 4; ++z) {
                v[8 * q + 2 * z] = __uint_as_float(wd[z] << 16);
                v[8 * q + 2 * z + 1] = __uint_as_float(wd[z] & 0xFFFF0000u);
              }
            }
          } else {
            const float* src = a.hin + size_t(row) * K + g0;
#pragma unroll
            for (int q = 0; q < Gm::G / 4; ++q) {
              const float4 u = __ldcg(reinterpret_cast<const float4*>(src + 4 * q));
              v[4 * q] = u.x; v[4 * q + 1] = u.y; v[4 * q + 2] = u.z; v[4 * q + 3] = u.w;
            }
          }
          uint4 parts[Gm::NPART];
          pack_int_order<BITS, Gm::G>(v, mul, parts);
          const int base = staged_offset<BITS, LPR, CPL>(g0);
#pragma unroll
          for (int part = 0; part < Gm::NPART; ++part) *reinterpret_cast<uint4*>(dst + base + part * LPR * 8) = parts[part];
        }
        if (lane == 0) {
          tok_inv[tl] = act_inv<BITS>(sh);
          tok_pos[tl] = p;
          tok_w[tl] = (MODE == DOWN && !is_shared) ? __ldcg(rv.topk_w + __ldcg(rv.pairs + p)) : 1.f;
        }
      }
      named_bar_sync(1, kNCW * 32);
    }

    const int slot = i % kStages;
    bool ok = !*abort_flag;
    if (ok && !mbar_wait(&full[slot], (i / kStages) & 1, abort_flag)) {
      ok = false;
      *abort_flag = 1;
      report_error(a.status, MOE_ERR_TIMEOUT, 3);
    }
    if (ok) {
      const unsigned char* st = ring + slot * Gm::STAGE_BYTES;
      Rows rows{st + rl0 * Gm::RB, st + Gm::CODE_BYTES + rl0 * (Gm::SPR >> PS) * SSZ, cur.stage * Gm::RPS + rl0,
                a.xk};
      if (SF) {
        const float* rsb = cur.e >= rv.E ? a.sh_row_scales : a.row_scales + size_t(cur.e) * a.rows;
        rows.rs0 = __ldg(rsb + rows.r0);
        rows.rs1 = __ldg(rsb + rows.r0 + 1);
      }
#pragma unroll 1
      for (int tb = 0; tb < nc; tb += NTB) {
        const int nt = min(NTB, nc - tb);          // warp-uniform
        if (nt == 1) rows_dot<MODE, BITS, LPR, CPL, 1, PS, SF>(a.out, a.out_cols, rows, xs + size_t(tb) * K, tb, lr, tok_inv, tok_w, tok_pos, 1);
        else if (nt == 2) rows_dot<MODE, BITS, LPR, CPL, 2, PS, SF>(a.out, a.out_cols, rows, xs + size_t(tb) * K, tb, lr, tok_inv, tok_w, tok_pos, 2);
        else rows_dot<MODE, BITS, LPR, CPL, 4, PS, SF>(a.out, a.out_cols, rows, xs + size_t(tb) * K, tb, lr, tok_inv, tok_w, tok_pos, nt);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
  }
}

// --------------------------------------------------------- dequant hook
// Writes out[r][j] = q * scale for rows row0.. of a packed matrix, with the
// byte and scale decoders the GEMV uses (q4_bytes / q2_bytes: signed bytes
// 16 q or 64 q; fp16 or E4M3 scales, the latter times the row's fp32 scale:
// q * e4m3 is exact, so the product is rounded once); test hook, not on the
// timed path.
template <int BITS, int SF>
__global__ void dequant_rows_kernel(const uint8_t* __restrict__ codes, const unsigned char* __restrict__ scales,
                                    const float* __restrict__ row_scales, int row0, int rows, int cols, int BLOCK,
                                    uint32_t xk, float* __restrict__ out) {
  constexpr int G = BITS == 4 ? 8 : 16;
  const int words_per_row = cols / G;
  const long long total = (long long)rows * words_per_row;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int r = int(i / words_per_row), wi = int(i % words_per_row);
    const size_t row = size_t(row0 + r);
    const uint32_t v = *reinterpret_cast<const uint32_t*>(codes + row * (cols * BITS / 8) + size_t(wi) * 4);
    uint32_t f[4];
    if (BITS == 4) {
      q4_bytes(v, xk, f[0], f[1]);
    } else {
      q2_bytes(v, xk, f);
    }
    for (int j = 0; j < G; ++j) {
      const int col = wi * G + j;
      // element j: 4-bit -> byte j/2 of lo (even j) / hi (odd j);
      //            2-bit -> byte j/4 of field j%4
      const uint32_t word = BITS == 4 ? f[j & 1] : f[j & 3];
      const int byte = BITS == 4 ? (j >> 1) : (j >> 2);
      const int qb = int(int8_t(uint8_t(word >> (8 * byte))));
      const size_t si = row * (cols / BLOCK) + col / BLOCK;
      if (SF) {
        out[size_t(r) * cols + col] = (ldexpf(float(qb), -CodeMul<BITS>::kLog2) * e4m3_value(scales[si])) * row_scales[row];
      } else {
        const float sc = __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(scales)[si]));
        out[size_t(r) * cols + col] = ldexpf(float(qb), -CodeMul<BITS>::kLog2) * sc;
      }
    }
  }
}

template <int BITS, int LPR, int CPL>
PassPlan plan_of(int rows, int K) {
  using Gm = Geom<BITS, LPR, CPL>;
  PassPlan p;
  p.spe = rows / Gm::RPS;
  const int avail = kSmemBudget - 256 - kStages * Gm::STAGE_BYTES - kMaxNTC * 12;
  p.ntc = min(kMaxNTC, (avail / (K * 2)) & ~1);
  return p;
}

template <int MODE, int BITS, int LPR, int CPL, int PS, int SF>
cudaError_t launch_one(FfnArgs fa, int num_sms, cudaStream_t s) {
  using Gm = Geom<BITS, LPR, CPL>;
  auto kern = ffn_tma_kernel<MODE, BITS, LPR, CPL, PS, SF>;
  const size_t smem = 256 + size_t(kStages) * Gm::STAGE_BYTES + size_t(fa.ntc) * Gm::K * 2 + kMaxNTC * 12;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  return launch_pdl(kern, dim3(num_sms), dim3(kThreads), smem, s, fa);
}

// 16-byte pieces per row C -> lanes per row (largest power of two <= 32
// dividing C) and pieces per lane.
#define MOE_C_CASES(X) X(2, 2, 1) X(4, 4, 1) X(8, 8, 1) X(12, 4, 3) X(16, 16, 1) X(24, 8, 3) \
                       X(32, 32, 1) X(48, 16, 3) X(64, 16, 4) X(96, 32, 3) X(128, 32, 4)

template <int MODE, int BITS>
cudaError_t dispatch(int K, FfnArgs fa, int num_sms, cudaStream_t s) {
  const int C = K * BITS / 8 / 16;
  switch (C) {
#define X(c, lpr, cpl)                                                              \
  case c:                                                                           \
    if constexpr (BITS == 4) {                                                      \
      if (fa.block == 128) return launch_one<MODE, BITS, lpr, cpl, 2, 0>(fa, num_sms, s); \
    }                                                                               \
    if (fa.sf) return launch_one<MODE, BITS, lpr, cpl, 0, 1>(fa, num_sms, s);       \
    return launch_one<MODE, BITS, lpr, cpl, 0, 0>(fa, num_sms, s);
    MOE_C_CASES(X)
#undef X
    default: return cudaErrorInvalidValue;
  }
}

template <int BITS>
bool plan_for(int rows, int K, PassPlan* p) {
  const int C = K * BITS / 8 / 16;
  switch (C) {
#define X(c, lpr, cpl) \
  case c: { using Gm = Geom<BITS, lpr, cpl>; if (rows % Gm::RPS) return false; *p = plan_of<BITS, lpr, cpl>(rows, K); return p->ntc >= 2; }
    MOE_C_CASES(X)
#undef X
    default: return false;
  }
}

bool plans(int bits, int H, int I, PassPlan* gu, PassPlan* dn) {
  if (bits == 4) return plan_for<4>(2 * I, H, gu) && plan_for<4>(H, I, dn);
  return plan_for<2>(2 * I, H, gu) && plan_for<2>(H, I, dn);
}

}  // namespace

bool decode_shape_supported(int bits, int H, int I) {
  PassPlan g, d;
  return plans(bits, H, I, &g, &d);
}

void decode_plans(const moe_config& c, PassPlan* gu, PassPlan* dn) { plans(c.bits, c.hidden, c.inter, gu, dn); }

cudaError_t launch_decode_ffn(const LayerArgs& a, cudaEvent_t between) {
  const moe_config& c = a.cfg;
  const int H = c.hidden, I = c.inter, bits = c.bits;
  PassPlan pg, pd;
  if (!plans(bits, H, I, &pg, &pd)) return cudaErrorInvalidValue;
  RouteView rv;
  rv.T = a.T; rv.k = c.top_k; rv.E = c.num_experts; rv.shared = c.shared_inter > 0 ? 1 : 0;
  rv.status = reinterpret_cast<const int*>(a.ws + a.L.status);
  rv.ulist = reinterpret_cast<const int*>(a.ws + a.L.ulist);
  rv.offsets = reinterpret_cast<const int*>(a.ws + a.L.offsets);
  rv.pairs = reinterpret_cast<const int*>(a.ws + a.L.pairs);
  rv.inv = reinterpret_cast<const int*>(a.ws + a.L.inv);
  rv.topk_w = reinterpret_cast<const float*>(a.ws + a.L.topk_w);

  FfnArgs g{};
  g.codes = a.w.gate_up_codes; g.scales = reinterpret_cast<const unsigned char*>(a.w.gate_up_scales);
  g.sh_codes = a.w.shared_gate_up_codes;
  g.sh_scales = reinterpret_cast<const unsigned char*>(a.w.shared_gate_up_scales);
  g.sf = c.scale_fmt; g.row_scales = a.w.gate_up_row_scales; g.sh_row_scales = a.w.shared_gate_up_row_scales;
  g.expert_code_bytes = size_t(2 * I) * H * bits / 8;
  g.expert_scale_count = size_t(2 * I) * (H / c.block);
  g.rows = 2 * I; g.out_cols = I; g.ntc = pg.ntc; g.block = c.block; g.xk = code_xor(bits, c.half_levels);
  g.xin = a.x; g.hin = nullptr;
  g.out = reinterpret_cast<float*>(a.ws + a.L.h);
  g.status = reinterpret_cast<int*>(a.ws + a.L.status);
  g.rv = rv;
  g.rv.woff = reinterpret_cast<const int*>(a.ws + a.L.woff_gu);
  cudaError_t err = bits == 4 ? dispatch<GATEUP, 4>(H, g, a.num_sms, a.stream)
                              : dispatch<GATEUP, 2>(H, g, a.num_sms, a.stream);
  if (err != cudaSuccess) return err;
  if (between) cudaEventRecord(between, a.stream);

  FfnArgs d{};
  d.codes = a.w.down_codes; d.scales = reinterpret_cast<const unsigned char*>(a.w.down_scales);
  d.sh_codes = a.w.shared_down_codes; d.sh_scales = reinterpret_cast<const unsigned char*>(a.w.shared_down_scales);
  d.sf = c.scale_fmt; d.row_scales = a.w.down_row_scales; d.sh_row_scales = a.w.shared_down_row_scales;
  d.expert_code_bytes = size_t(H) * I * bits / 8;
  d.expert_scale_count = size_t(H) * (I / c.block);
  d.rows = H; d.out_cols = H; d.ntc = pd.ntc; d.block = c.block; d.xk = code_xor(bits, c.half_levels);
  d.xin = nullptr; d.hin = reinterpret_cast<const float*>(a.ws + a.L.h);
  d.out = reinterpret_cast<float*>(a.ws + a.L.y);
  d.status = reinterpret_cast<int*>(a.ws + a.L.status);
  d.rv = rv;
  d.rv.woff = reinterpret_cast<const int*>(a.ws + a.L.woff_dn);
  return bits == 4 ? dispatch<DOWN, 4>(I, d, a.num_sms, a.stream) : dispatch<DOWN, 2>(I, d, a.num_sms, a.stream);
}

cudaError_t launch_dequant_rows(int bits, int block, int half_levels, int scale_fmt, const uint8_t* codes,
                                const void* scales, const float* row_scales, int row0, int rows, int cols,
                                float* out, cudaStream_t s) {
  const int G = bits == 4 ? 8 : 16;
  const long long total = (long long)rows * (cols / G);
  const long long want = (total + 255) / 256;
  const int blocks = int(want < 4096 ? want : 4096);
  const uint32_t xk = code_xor(bits, half_levels);
  const unsigned char* sc = static_cast<const unsigned char*>(scales);
  if (bits == 4) {
    if (scale_fmt) dequant_rows_kernel<4, 1><<<blocks, 256, 0, s>>>(codes, sc, row_scales, row0, rows, cols, block, xk, out);
    else dequant_rows_kernel<4, 0><<<blocks, 256, 0, s>>>(codes, sc, row_scales, row0, rows, cols, block, xk, out);
  } else {
    if (scale_fmt) dequant_rows_kernel<2, 1><<<blocks, 256, 0, s>>>(codes, sc, row_scales, row0, rows, cols, block, xk, out);
    else dequant_rows_kernel<2, 0><<<blocks, 256, 0, s>>>(codes, sc, row_scales, row0, rows, cols, block, xk, out);
  }
  return cudaGetLastError();
}

}  // namespace moe
