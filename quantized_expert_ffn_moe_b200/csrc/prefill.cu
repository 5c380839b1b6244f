// Prefill path (many tokens per expert): grouped GEMMs on the tcgen05 tensor
// cores with the packed weights dequantized into shared memory.
//
// Same operation as the decode path (the expert FFN that replaces the dense
// FFN, "Running a 125B Model on a Single RTX 5090: Strata Benchmarks Qwen3.8
// Flash Next", section "Layer 1: On-Demand MoE Expert Scheduling"); with tens
// of tokens per expert every weight byte feeds enough multiply-adds for the
// work to be a dense contraction, so it runs on the tensor cores.
//
// Per tile (expert e, 128 weight rows, up to 128 of e's tokens):
//   D[128 x N] (fp32, TMEM) = W_e[rows, :] (fp16, dequantized) . X_e^T (fp16)
// with the weights as the UMMA A operand (M = 128) and the tokens as B (N =
// the tile's token count rounded up to 16), K in steps of 64.
// Warp roles of the persistent CTA (one per SM):
//   warp 0      TMA of packed codes + fp16 scales (2-D tensor maps, swizzled)
//   warp 1      TMA of the token tile (SWIZZLE_128B, the UMMA K-major layout)
//   warp 2      TMEM allocation; one thread issues tcgen05.mma + commits
//   warps 3-10  dequantize codes into the fp16 A operand, written straight
//               into tensor memory (tcgen05.st, one row per TMEM lane), so
//               the dequantized tile never passes through shared memory
//   warps 11-14 epilogue: tcgen05.ld from TMEM, SwiGLU (gate/up) or gate
//               weight (down), stores
// Operands are fp16: a weight is q * s rounded once (q exact, s the block's
// fp16 scale); token rows are converted exactly after a per-token power of
// two brings their largest element into [2^13, 2^14); h is kept in fp16
// between the passes.  Within a group of 8 (4-bit) or 16 (2-bit) consecutive
// k the dequantizer emits elements in the pair order of its integer decode, so
// the token operand is stored with the same permutation of k (the contraction
// is unchanged).  Every wait is bounded.
#include "moe_internal.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

namespace moe {

namespace {

constexpr int PBM = 128;       // weight rows per tile
constexpr int PBN = kPrefillTileN;   // tokens per tile (max)
static_assert(PBN == 128, "the grouping kernel's tile prefix assumes 128 tokens per tile");
constexpr int PBK = 64;        // k of one 128-byte swizzle row of fp16 (a TMA box; the router GEMM's stage)
constexpr int PSK = 128;       // grouped GEMM: k per A/B stage (two swizzle atoms, 8 MMAs per barrier)
constexpr int RAWK = 256;      // k per packed stage
constexpr int PNK = 4;         // A (tensor memory) / B (shared memory) stages
constexpr int PNR = 4;         // packed stages
constexpr int kWarpRaw = 0, kWarpB = 1, kWarpMma = 2, kWarpDq0 = 3, kNumDq = 8, kWarpEp0 = 11;
// Epilogue warps: two per tensor-memory lane quarter for the down GEMM, whose
// tiles carry only I / 128 k-blocks of MMAs and whose epilogue writes a value
// per (row, token); one per quarter for gate/up (sixteen k-blocks per tile,
// and its register budget does not fit 19 warps).
template <int MODE> struct PEp {
  static constexpr int kNum = MODE == 1 ? 8 : 4;
  static constexpr int kThreads = (kWarpEp0 + kNum) * 32;
};
constexpr uint32_t kTmemCols = 2 * PBN;          // router GEMM: two accumulators
// Grouped GEMM tensor memory: two accumulators of PBN columns, then PNK
// dequantized A stages of PSK / 2 columns (128 lanes = the tile's rows, two
// fp16 per 32-bit column in k order).
constexpr uint32_t kAColBase = 2 * PBN;
constexpr uint32_t kAStageCols = PSK / 2;
constexpr uint32_t kPTmemCols = 512;
static_assert(kAColBase + PNK * kAStageCols <= kPTmemCols, "tensor memory budget");
// barriers (2 PNR + 2 PNK + 4 of 8 bytes), the TMEM address and the abort flag
constexpr int kBarBytes = 512;
static_assert((2 * PNR + 2 * PNK + 4) * 8 + 8 <= kBarBytes, "barrier area");
constexpr int kTileTab = 512;      // per-CTA tile table entries (16 B each)
constexpr int kAStageBytes = PBM * 128;           // 16 KB (router GEMM)
constexpr int kBStageBytes = PBN * 128;           // 16 KB: one swizzle atom column of the token tile
constexpr int kGBStageBytes = kBStageBytes * (PSK / PBK);   // grouped GEMM token stage

template <int BITS>
struct PGeom {
  static constexpr int BLOCK = BITS == 4 ? 32 : 16;
  static constexpr int IB = RAWK * BITS / 8;              // packed bytes of a row per packed stage
  static constexpr int SB = RAWK / BLOCK * 2;             // scale bytes of a row per packed stage
  static constexpr int CODE_BYTES = PBM * IB;
  static constexpr int SCALE_BYTES = PBM * SB;
  static constexpr int SCALE_OFF = (CODE_BYTES + 1023) / 1024 * 1024;   // swizzled scales need alignment
  static constexpr int RAW_BYTES = SCALE_OFF + SCALE_BYTES;
  static constexpr int G = BITS == 4 ? 8 : 16;            // k group of the pair order
};

struct PrefillArgs {
  int K;                  // reduction length (H gate/up, I down)
  int rows_pe;            // weight rows per expert (2I gate/up, H down)
  int out_cols;           // I (h) or H (Y)
  RouteView rv;
  const int* ntoff;       // [nslots+1] prefix of token tiles per slot
  uint16_t* hout;         // gate/up: h [P][I] fp16 bits, k permuted for the down pass
  const float* xinv;      // gate/up: [P] inverse power-of-two scale of each token row
  uint16_t* yout;         // down: Y [P][H] fp16 bits (gate weight applied)
  int* status;
  unsigned long long* timing;   // null, or [gridDim][16] per-role wait times (ns) of this launch
  int gated;                    // 1: no tiles unless the fused decode kernel handed the layer over
  int half_levels;              // 1: codes are the half-integer levels q = c - (2^bits - 1)/2
};

constexpr int kPTime = 16;

// ------------------------------------------------------------ primitives
// The same with an L2 cache policy (the packed weights: read once per tile).
__device__ __forceinline__ void tma_load_2d_hint(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar,
                                                 uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar)),
        "l"(policy)
      : "memory");
}
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Same with the A operand in tensor memory (lane = row, two fp16 per column).
__device__ __forceinline__ void tc_mma_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// True in exactly one lane of a fully active warp (elect.sync).
__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}" : "=r"(pred));
  return pred != 0;
}
// 32 consecutive columns of this thread's tensor-memory lane (warp-wide; the
// warp's lane quarter is fixed by its rank within the warpgroup).
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t v[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
      ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]),
        "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]),
        "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// UMMA shared-memory descriptor of a K-major SWIZZLE_128B tile: rows of 128 B,
// 8-row atoms 1024 B apart (SBO), version 1, layout type 2.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return uint64_t((saddr & 0x3FFFF) >> 4) | (uint64_t(1) << 16) | (uint64_t(1024 >> 4) << 32) |
         (uint64_t(1) << 46) | (uint64_t(2) << 61);
}
// Instruction descriptor: D fp32, A and B fp16, both K-major, M = 128, N.
__device__ __forceinline__ uint32_t idesc_f16(int n) {
  return (1u << 4) | (uint32_t(n >> 3) << 17) | (uint32_t(PBM >> 4) << 24);
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t v[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t v[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
        "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
        "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Packed word -> fp16 pairs q * s (q exact from the magic-number decode, one
// rounding in the multiply).  Pair order as in the decode path: 4-bit
// (q_j, q_{j+4}), 2-bit (q_j, q_{j+8}).  half: the half-integer levels.
__device__ __forceinline__ void dq4_f16(uint32_t v, __half2 s, bool half, uint32_t out[4]) {
  __half2 q[4];
  if (half) decode_q4x8_half(v, q);
  else decode_q4x8(v, q);
#pragma unroll
  for (int j = 0; j < 4; ++j) out[j] = h2_as_u32(__hmul2(q[j], s));
}
__device__ __forceinline__ void dq2_f16(uint32_t v, __half2 s, bool half, uint32_t out[8]) {
  __half2 q[8];
  if (half) decode_q2x16_half(v, q);
  else decode_q2x16(v, q);
#pragma unroll
  for (int j = 0; j < 8; ++j) out[j] = h2_as_u32(__hmul2(q[j], s));
}

// mbar_wait that adds the SM cycles it waited to *acc when acc is non-null.
__device__ __forceinline__ bool mbar_wait_t(uint64_t* bar, uint32_t parity, const volatile int* abort_flag,
                                            unsigned long long* acc) {
  if (!acc) return mbar_wait(bar, parity, abort_flag);
  const long long t0 = clock64();
  const bool ok = mbar_wait(bar, parity, abort_flag);
  *acc += clock64() - t0;
  return ok;
}

struct TileInfo {
  int slot, e, p0, n, nvalid, m, j;
};

// Slot table of the pass in shared memory (read once per CTA): token-tile
// prefix, expert, first routed position and token count of every slot.
struct SlotTab {
  int* ntoff;   // [nslots + 1]
  int* e;       // [nslots]
  int* p0;      // [nslots]
  int* n;       // [nslots]
};

__device__ __forceinline__ void tile_info(const SlotTab& st, int nslots, int mt, int t, TileInfo* ti) {
  const int g = t / mt;
  ti->m = t % mt;
  int lo = 0, hi = nslots - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (st.ntoff[mid] <= g) lo = mid; else hi = mid - 1;
  }
  ti->slot = lo;
  ti->j = g - st.ntoff[lo];
  ti->e = st.e[lo];
  ti->p0 = st.p0[lo];
  ti->n = st.n[lo];
  ti->nvalid = min(PBN, ti->n - ti->j * PBN);
}

template <int MODE, int BITS>
__global__ void __launch_bounds__(PEp<MODE>::kThreads, 1) prefill_gemm_kernel(
    PrefillArgs a, const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_scales,
    const __grid_constant__ CUtensorMap tm_sh_codes, const __grid_constant__ CUtensorMap tm_sh_scales,
    const __grid_constant__ CUtensorMap tm_b) {
  using Gm = PGeom<BITS>;
  extern __shared__ __align__(1024) unsigned char psmem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(psmem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sB = base;                                   // PNK x 32 KB
  unsigned char* sRaw = sB + PNK * kGBStageBytes;             // PNR x RAW_BYTES (1024-aligned each)
  constexpr int RAW_STRIDE = (Gm::RAW_BYTES + 1023) / 1024 * 1024;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sRaw + PNR * RAW_STRIDE);
  uint64_t* full_raw = bars;
  uint64_t* empty_raw = full_raw + PNR;
  uint64_t* full_a = empty_raw + PNR;
  uint64_t* empty_ab = full_a + PNK;
  uint64_t* acc_full = empty_ab + PNK;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < PNR; ++i) { mbar_init(&full_raw[i], 1); mbar_init(&empty_raw[i], kNumDq); }
    // full_a: the four dequant warps of the k-block's half + the token tile's bytes
    for (int i = 0; i < PNK; ++i) { mbar_init(&full_a[i], kNumDq / 2 + 1); mbar_init(&empty_ab[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&acc_full[i], 1); mbar_init(&acc_empty[i], PEp<MODE>::kNum); }
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == kWarpMma) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kPTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  pdl_wait();                     // tokens (and routing) come from earlier kernels
  pdl_launch_dependents();
  unsigned long long* tm = a.timing ? a.timing + size_t(blockIdx.x) * kPTime : nullptr;
  unsigned long long tw0 = 0, tw1 = 0, tw2 = 0, tw3 = 0, tw4 = 0;   // this thread's totals (timed roles only)
  const unsigned long long t_start = tm ? global_ns() : 0;

  const RouteView& rv = a.rv;
  const bool closed = a.gated && __ldcg(rv.status + ST_PATH) == 0;     // the fused decode kernel kept the layer
  const int nslots = closed ? 0 : __ldcg(rv.status + ST_UCOUNT) + rv.shared;
  const int mt = a.rows_pe / PBM;
  // slot table into shared memory (nslots <= E + 1): one L2 round trip here
  // instead of a dependent binary search through global memory per tile
  SlotTab stab;
  stab.ntoff = reinterpret_cast<int*>(reinterpret_cast<unsigned char*>(bars) + kBarBytes);
  stab.e = stab.ntoff + (rv.E + 2);
  stab.p0 = stab.e + (rv.E + 1);
  stab.n = stab.p0 + (rv.E + 1);
  for (int i = threadIdx.x; i <= nslots; i += blockDim.x) {
    stab.ntoff[i] = __ldcg(a.ntoff + i);
    if (i < nslots) slot_range(rv, i, &stab.e[i], &stab.p0[i], &stab.n[i]);
  }
  __syncthreads();
  const int ntiles = closed ? 0 : stab.ntoff[nslots] * mt;
  const int KB = a.K / PSK, KR = a.K / RAWK;
  // this CTA's tiles (t = blockIdx.x + i * gridDim.x) decoded once into a
  // shared table, read by every role; beyond kTileTab tiles the lookup is redone
  int4* ttab = reinterpret_cast<int4*>((reinterpret_cast<uintptr_t>(stab.n + rv.E + 1) + 15) & ~uintptr_t(15));
  {
    const int my_tiles = ntiles > int(blockIdx.x) ? (ntiles - int(blockIdx.x) + int(gridDim.x) - 1) / int(gridDim.x) : 0;
    for (int i = threadIdx.x; i < min(my_tiles, kTileTab); i += blockDim.x) {
      TileInfo ti;
      tile_info(stab, nslots, mt, blockIdx.x + i * gridDim.x, &ti);
      ttab[i] = make_int4(ti.e, ti.p0, (ti.j << 16) | ti.m, ti.nvalid);
    }
  }
  __syncthreads();
  // tile i of this CTA (global tile t = blockIdx.x + i * gridDim.x)
  auto get_tile = [&](int i, TileInfo* ti) {
    if (i < kTileTab) {
      const int4 v = ttab[i];
      ti->e = v.x;
      ti->p0 = v.y;
      ti->j = v.z >> 16;
      ti->m = v.z & 0xFFFF;
      ti->nvalid = v.w;
    } else {
      tile_info(stab, nslots, mt, int(blockIdx.x) + i * int(gridDim.x), ti);
    }
  };

  if (warp == kWarpRaw && lane == 0) {
    // ------------------------------------------------ packed weight producer
    int rc = 0;
    for (int t = blockIdx.x, i = 0; t < ntiles && !*abort_flag; t += gridDim.x, ++i) {
      TileInfo ti;
      get_tile(i, &ti);
      const bool sh = ti.e >= rv.E;
      const CUtensorMap* mc = sh ? &tm_sh_codes : &tm_codes;
      const CUtensorMap* ms = sh ? &tm_sh_scales : &tm_scales;
      const int row = (sh ? 0 : ti.e * a.rows_pe) + ti.m * PBM;
      for (int r = 0; r < KR; ++r, ++rc) {
        const int s = rc % PNR;
        if (rc >= PNR && !mbar_wait_t(&empty_raw[s], ((rc / PNR) - 1) & 1, abort_flag, tm ? &tw0 : nullptr)) {
          *abort_flag = 1; report_error(a.status, MOE_ERR_TIMEOUT, 10); break;
        }
        unsigned char* dst = sRaw + s * RAW_STRIDE;
        mbar_arrive_expect_tx(&full_raw[s], Gm::CODE_BYTES + Gm::SCALE_BYTES);
        if (ti.n <= kPrefillTileN) {
          // one token tile: these weight bytes are read once in the pass
          const uint64_t pol = l2_evict_first_policy();
          tma_load_2d_hint(dst, mc, r * Gm::IB, row, &full_raw[s], pol);
          tma_load_2d_hint(dst + Gm::SCALE_OFF, ms, r * (RAWK / Gm::BLOCK), row, &full_raw[s], pol);
        } else {
          tma_load_2d(dst, mc, r * Gm::IB, row, &full_raw[s]);
          tma_load_2d(dst + Gm::SCALE_OFF, ms, r * (RAWK / Gm::BLOCK), row, &full_raw[s]);
        }
      }
    }
    for (int i = max(0, rc - PNR); i < rc; ++i)
      if (!mbar_wait(&full_raw[i % PNR], (i / PNR) & 1, nullptr)) report_error(a.status, MOE_ERR_TIMEOUT, 11);
    if (tm) tm[0] = tw0;
  } else if (warp == kWarpB && lane == 0) {
    // ------------------------------------------------------ token producer
    int kc = 0;
    for (int t = blockIdx.x, i = 0; t < ntiles && !*abort_flag; t += gridDim.x, ++i) {
      TileInfo ti;
      get_tile(i, &ti);
      const int prow = ti.p0 + ti.j * PBN;
      for (int kb = 0; kb < KB; ++kb, ++kc) {
        const int s = kc % PNK;
        if (kc >= PNK && !mbar_wait_t(&empty_ab[s], ((kc / PNK) - 1) & 1, abort_flag, tm ? &tw0 : nullptr)) {
          *abort_flag = 1; report_error(a.status, MOE_ERR_TIMEOUT, 12); break;
        }
        mbar_arrive_expect_tx(&full_a[s], kGBStageBytes);
#pragma unroll
        for (int h = 0; h < PSK / PBK; ++h)
          tma_load_2d(sB + s * kGBStageBytes + h * kBStageBytes, &tm_b, kb * PSK + h * PBK, prow, &full_a[s]);
      }
    }
    for (int i = max(0, kc - PNK); i < kc; ++i)
      if (!mbar_wait(&full_a[i % PNK], (i / PNK) & 1, nullptr)) report_error(a.status, MOE_ERR_TIMEOUT, 13);
    if (tm) tm[1] = tw0;
  } else if (warp == kWarpMma) {
    // ---------------------------------------------------------------- MMA
    // The whole warp runs this loop, so its control and every MMA operand are
    // warp-uniform; one elected lane issues each stage's MMAs and commit.  (A
    // single-lane loop left the operands per-thread: its issue competed with
    // the dequant warps and cost ~90 instead of ~55-70 cycles per MMA.)
    int kc = 0, tc = 0;
    const long long c_start = tm ? clock64() : 0;
    bool ok = true;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++tc) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
      const long long cti = tm ? clock64() : 0;
      TileInfo ti;
      get_tile(tc, &ti);
      if (tm) tw4 += clock64() - cti;
      const int buf = tc & 1;
      if (tc >= 2) {
        const long long cw = tm ? clock64() : 0;
        ok = __all_sync(0xffffffffu, mbar_wait(&acc_empty[buf], ((tc >> 1) - 1) & 1, abort_flag));
        if (tm) tw2 += clock64() - cw;
      }
      if (!ok) {
        if (lane == 0) { *abort_flag = 1; report_error(a.status, MOE_ERR_TIMEOUT, 14); }
        break;
      }
      tc_fence_after();
      const uint32_t idesc = idesc_f16((ti.nvalid + 15) & ~15);
      const uint32_t d_tmem = tmem_base + uint32_t(buf * PBN);
      for (int kb = 0; kb < KB; ++kb, ++kc) {
        const int s = kc % PNK;
        const long long cw = tm ? clock64() : 0;
        ok = __all_sync(0xffffffffu, mbar_wait(&full_a[s], (kc / PNK) & 1, abort_flag));
        if (!ok) {
          if (lane == 0) { *abort_flag = 1; report_error(a.status, MOE_ERR_TIMEOUT, 15); }
          break;
        }
        const long long ci = tm ? clock64() : 0;
        if (tm) tw0 += ci - cw;
        tc_fence_after();
        const uint32_t a0 = tmem_base + kAColBase + uint32_t(s) * kAStageCols;
        const uint64_t bd = sw128_desc(smem_u32(sB + s * kGBStageBytes));
        if (elect_one()) {
#pragma unroll
          for (int k = 0; k < PSK / 16; ++k)
            tc_mma_ta(d_tmem, a0 + uint32_t(k * 8), bd + uint64_t(((k >> 2) * kBStageBytes + (k & 3) * 32) >> 4),
                      idesc, (kb | k) ? 1u : 0u);
          tc_commit(&empty_ab[s]);
          if (kb == KB - 1) tc_commit(&acc_full[buf]);
        }
        __syncwarp();
        if (tm) tw3 += clock64() - ci;
      }
      if (!ok) break;
    }
    // wait for the last MMAs before the CTA tears down TMEM
    if (kc > 0 && !__all_sync(0xffffffffu, mbar_wait(&empty_ab[(kc - 1) % PNK], ((kc - 1) / PNK) & 1, nullptr)) &&
        lane == 0)
      report_error(a.status, MOE_ERR_TIMEOUT, 16);
    if (tm && lane == 0) { tm[2] = tw0; tm[3] = tw1; tm[4] = tw2; tm[8] = t_start; tm[9] = global_ns(); tm[10] = tc; tm[12] = tw3; tm[13] = tw4; tm[14] = kc; tm[15] = clock64() - c_start; }
  } else if (warp >= kWarpDq0 && warp < kWarpDq0 + kNumDq) {
    // ----------------------------------------------------------- dequant
    // warp w writes rows of its tensor-memory lane quarter (w % 4); the two
    // warps of a quarter take the first and second half of a packed stage
    const int r = (warp & 3) * 32 + lane;          // tile row
    const bool hl = a.half_levels != 0;
    const int half = (warp - kWarpDq0) >> 2;       // which of the two A stages of a packed stage
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    static_assert(RAWK == 2 * PSK, "a packed stage feeds two A stages, one per dequant half");
    int rc = 0, kc = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
      for (int rs = 0; rs < KR; ++rs, ++rc) {
        const int s = rc % PNR;
        const bool timed = tm && threadIdx.x == kWarpDq0 * 32;
        bool ok = !*abort_flag && mbar_wait_t(&full_raw[s], (rc / PNR) & 1, abort_flag, timed ? &tw0 : nullptr);
        const unsigned char* raw = sRaw + s * RAW_STRIDE;
        const unsigned char* sc = raw + Gm::SCALE_OFF;
        const int kglob = kc + half;                // global counter of this thread's A/B stage
        const int as = kglob % PNK;
        if (ok && kglob >= PNK) ok = mbar_wait_t(&empty_ab[as], ((kglob / PNK) - 1) & 1, abort_flag, timed ? &tw1 : nullptr);
        ok = __all_sync(0xffffffffu, ok);           // the tensor-memory store is warp-wide
        if (ok) {
          tc_fence_after();
          // the row's 128 fp16 of this A stage, in k order, in two 64-column halves
#pragma unroll
          for (int hb = 0; hb < 2; ++hb) {
            const int kbl = half * 2 + hb;          // 64-k block within the packed stage (0..3)
            uint32_t o32[32];
            if (BITS == 4) {
              // 2 x 16 bytes of codes = 64 weights, 2 scales
#pragma unroll
              for (int cc = 0; cc < 2; ++cc) {
                const int lc = kbl * 2 + cc;                     // logical 16-B chunk in the 128-B row
                const uint4 w = *reinterpret_cast<const uint4*>(raw + r * Gm::IB + ((lc ^ (r & 7)) << 4));
                const __half hs = *reinterpret_cast<const __half*>(sc + r * Gm::SB + lc * 2);
                const __half2 s2 = __half2half2(hs);
                const uint32_t wd[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) dq4_f16(wd[q], s2, hl, o32 + (cc * 4 + q) * 4);
              }
            } else {
              // 16 bytes of codes = 64 weights in 4 words, 4 scales
              const int lc = kbl;                                // logical 16-B chunk in the 64-B row
              const uint4 w = *reinterpret_cast<const uint4*>(raw + r * Gm::IB + ((lc ^ ((r >> 1) & 3)) << 4));
              const int sci = kbl * 4;                           // first scale of this block (of 16 per row)
              const int schunk = sci >> 3;                       // logical 16-B chunk of the 32-B scale row
              const uint4 sv = *reinterpret_cast<const uint4*>(sc + r * Gm::SB + ((schunk ^ ((r >> 2) & 1)) << 4));
              const uint32_t svw[4] = {sv.x, sv.y, sv.z, sv.w};
              const uint32_t wd[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const int si = (sci & 7) + q;                    // scale index within the 16-B chunk
                const uint32_t pr = svw[si >> 1];
                const __half hs = __ushort_as_half((unsigned short)((si & 1) ? (pr >> 16) : (pr & 0xFFFFu)));
                const __half2 s2 = __half2half2(hs);
                dq2_f16(wd[q], s2, hl, o32 + q * 8);
              }
            }
            tmem_st32(tmem_base + lane_base + kAColBase + uint32_t(as) * kAStageCols + uint32_t(hb * 32), o32);
          }
          tmem_st_wait();
          tc_fence_before();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&full_a[as]);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_raw[s]);
        if (!ok && !*abort_flag) { *abort_flag = 1; report_error(a.status, MOE_ERR_TIMEOUT, 17); }
        kc += 2;
      }
    }
    if (tm && threadIdx.x == kWarpDq0 * 32) { tm[5] = tw0; tm[6] = tw1; }
  } else if (warp >= kWarpEp0 && warp < kWarpEp0 + PEp<MODE>::kNum) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                         // TMEM lane quarter of this warp
    const int r = q * 32 + lane;                    // tile row
    constexpr int kColStep = 32 * (PEp<MODE>::kNum / 4);
    const int c_first = ((warp - kWarpEp0) >> 2) * 32;   // the warps of a quarter take alternate 32-column chunks
    // per-column factors of a tile (gate/up: the token row's inverse scale,
    // down: the gate weight), column u*32 + lane in f[u].  They are fetched
    // one tile ahead (down: the pair ids while the current tile's columns are
    // written, the gate weights after), so their latency overlaps the work.
    auto first_level = [&](const TileInfo& tn, float fo[PBN / 32], int po[PBN / 32]) {
      const int prn = tn.p0 + tn.j * PBN;
      const bool shn = tn.e >= rv.E;
#pragma unroll
      for (int u = 0; u < PBN / 32; ++u) {
        const int c = u * 32 + lane;
        fo[u] = 1.f;
        po[u] = -1;
        if (c < tn.nvalid) {
          if (MODE == 0) fo[u] = __ldg(a.xinv + prn + c);
          else if (!shn) po[u] = __ldg(rv.pairs + prn + c);
        }
      }
    };
    auto second_level = [&](float fo[PBN / 32], const int po[PBN / 32]) {
      if (MODE == 1) {
#pragma unroll
        for (int u = 0; u < PBN / 32; ++u)
          if (po[u] >= 0) fo[u] = __ldg(rv.topk_w + po[u]);
      }
    };
    int tc = 0;
    TileInfo ti_n;
    float f_n[PBN / 32];
    int pr_n[PBN / 32];
    if (blockIdx.x < ntiles) {
      get_tile(0, &ti_n);
      first_level(ti_n, f_n, pr_n);
      second_level(f_n, pr_n);
    }
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++tc) {
      const TileInfo ti = ti_n;
      float f[PBN / 32];
#pragma unroll
      for (int u = 0; u < PBN / 32; ++u) f[u] = f_n[u];
      const int buf = tc & 1;
      const int R = ti.m * PBM + r;                 // row of the expert matrix
      const int prow = ti.p0 + ti.j * PBN;
      const bool timed = tm && threadIdx.x == kWarpEp0 * 32;
      if (*abort_flag || !mbar_wait_t(&acc_full[buf], (tc >> 1) & 1, abort_flag, timed ? &tw0 : nullptr)) {
        if (!*abort_flag) { *abort_flag = 1; report_error(a.status, MOE_ERR_TIMEOUT, 18); }
        break;
      }
      const bool more = t + int(gridDim.x) < ntiles;
      if (more) {
        get_tile(tc + 1, &ti_n);
        first_level(ti_n, f_n, pr_n);
      }
      tc_fence_after();
      for (int n0 = c_first; n0 < ti.nvalid; n0 += kColStep) {
        uint32_t v[32];
        tmem_ld32(tmem_base + (uint32_t(q * 32) << 16) + uint32_t(buf * PBN + n0), v);
        const int u0 = n0 >> 5;
        const float colf = u0 == 0 ? f[0] : u0 == 1 ? f[1] : u0 == 2 ? f[2] : f[3];
        if (MODE == 0) {
          // rows alternate gate / up: lane pairs (2i, 2i+1) hold g and u of row
          // pair i.  For columns (c, c+1) the even lane takes column c and the
          // odd lane column c+1 (one exchange), so both lanes do the SwiGLU.
          const int i = R >> 1;
          const int G = Gm::G;
          const int ip = (i & ~(G - 1)) | decode_slot(BITS, i & (G - 1));
          const int odd = lane & 1;
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const float mine = __uint_as_float(v[c + odd]);
            const float other = __shfl_xor_sync(0xffffffffu, __uint_as_float(v[c + 1 - odd]), 1);
            const int col = c + odd;
            const float xi = __shfl_sync(0xffffffffu, colf, col);
            if (n0 + col < ti.nvalid) {
              const float g = (odd ? other : mine) * xi, u = (odd ? mine : other) * xi;
              const float hval = __fdividef(g * u, 1.f + __expf(-g));
              a.hout[size_t(prow + n0 + col) * a.out_cols + ip] = __half_as_ushort(__float2half_rn(hval));
            }
          }
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float w = __shfl_sync(0xffffffffu, colf, c);
            if (n0 + c < ti.nvalid)
              a.yout[size_t(prow + n0 + c) * a.out_cols + R] = __half_as_ushort(__float2half_rn(__uint_as_float(v[c]) * w));
          }
        }
      }
      if (more) second_level(f_n, pr_n);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
    }
    if (tm && threadIdx.x == kWarpEp0 * 32) { tm[7] = tw0; tm[11] = global_ns(); }
  }

  // ----------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kPTmemCols) : "memory");
  }
}

// 1-D bulk copy from shared to global memory (both addresses 16-byte aligned,
// bytes a multiple of 16), in this thread's bulk async-group.
__device__ __forceinline__ void bulk_s2g(void* gdst, const void* ssrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(smem_u32(ssrc)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Until this thread's bulk copies have read their shared-memory sources.
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Until this thread's bulk copies have completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Shared-memory stores of this thread made visible to the bulk-copy (async) proxy.
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Token rows scattered into expert order as fp16 (routed positions, then the
// shared expert's): one warp per token converts its row once -- exactly, after
// the power of two that brings its largest magnitude into [2^13, 2^14), with k
// permuted within each group of 8 (4-bit) / 16 (2-bit) to match the
// dequantizer's pair order -- into its row of shared memory, and one lane
// copies that row in bulk to every position of the token (inv[t k + j],
// position -1 = another rank's expert; T k + t for the shared expert), with
// xinv = the inverse power of two.  Dynamic shared memory: 8 rows of H fp16.
template <int BITS>
__global__ void __launch_bounds__(256) gather_tokens_kernel(const uint16_t* __restrict__ x, RouteView rv, int H,
                                                            uint16_t* __restrict__ xs, float* __restrict__ xinv,
                                                            int gated) {
  pdl_wait();
  pdl_launch_dependents();
  if (gated && __ldcg(rv.status + ST_PATH) == 0) return;     // the fused decode kernel kept the layer
  constexpr int G = BITS == 4 ? 8 : 16;
  constexpr int kMaxChunks = 4096 / (32 * G);              // chunks of G elements per lane (H <= 4096)
  extern __shared__ __align__(16) unsigned char gsm[];
  const int lane = threadIdx.x & 31;
  uint16_t* srow = reinterpret_cast<uint16_t*>(gsm) + size_t(threadIdx.x >> 5) * H;
  for (int tok = blockIdx.x * 8 + (threadIdx.x >> 5); tok < rv.T; tok += gridDim.x * 8) {
    const uint16_t* src = x + size_t(tok) * H;
    float vmax = 0.f;
    for (int h0 = lane * 8; h0 < H; h0 += 256) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + h0));
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int z = 0; z < 4; ++z)
        vmax = fmaxf(vmax, fmaxf(fabsf(__uint_as_float(w[z] << 16)), fabsf(__uint_as_float(w[z] & 0xFFFF0000u))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
    int sh = 0;
    if (vmax > 0.f) {
      int ex;
      frexpf(vmax, &ex);
      sh = min(max(14 - ex, -100), 100);
    }
    const float mul = ldexpf(1.f, sh), inv_mul = ldexpf(1.f, -sh);
    // the converted row, chunk c of this lane = elements (c * 32 + lane) * G ...
    // (H = 256 at 2-bit: 16 chunks of 16, half the lanes hold one)
    uint4 row[kMaxChunks][G / 8];
#pragma unroll
    for (int c = 0; c < kMaxChunks; ++c) {
      const int h0 = (c * 32 + lane) * G;
      if (c * 32 * G >= H) break;
      if (h0 >= H) continue;
      float in[G];
#pragma unroll
      for (int q = 0; q < G / 8; ++q) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + h0 + 8 * q));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int z = 0; z < 4; ++z) {
          in[8 * q + 2 * z] = __uint_as_float(w[z] << 16);
          in[8 * q + 2 * z + 1] = __uint_as_float(w[z] & 0xFFFF0000u);
        }
      }
      pack_pair_order<G>(in, mul, row[c]);
    }
    // the warp's row buffer is free again once the previous token's copies
    // have read it
    if (lane == 0) bulk_wait_read_all();
    __syncwarp();
#pragma unroll
    for (int c = 0; c < kMaxChunks; ++c) {
      const int h0 = (c * 32 + lane) * G;
      if (c * 32 * G >= H) break;
      if (h0 >= H) continue;
#pragma unroll
      for (int q = 0; q < G / 8; ++q) *reinterpret_cast<uint4*>(srow + h0 + 8 * q) = row[c][q];
    }
    fence_proxy_async_smem();
    __syncwarp();
    // every position of the token: its k routed pairs, then the shared expert
    if (lane == 0) {
      const int np = rv.k + (rv.shared ? 1 : 0);
      for (int j = 0; j < np; ++j) {
        const int p = j < rv.k ? __ldg(rv.inv + size_t(tok) * rv.k + j) : rv.T * rv.k + tok;
        if (p < 0) continue;                                 // another rank's expert
        bulk_s2g(xs + size_t(p) * H, srow, uint32_t(H) * 2);
        xinv[p] = inv_mul;
      }
      bulk_commit();
    }
  }
  // the rows are in global memory before the warp (and its shared memory) goes
  if (lane == 0) bulk_wait_all();
}

// Router logits of a large batch on the tensor cores:
//   logits[t][e] = sum_h x[t][h] Wr[e][h] (+ b[e])
// D[128 experts x N tokens] in TMEM from bf16 A = router rows and B = token
// rows (both by TMA, SWIZZLE_128B), fp32 accumulation; bf16 x bf16 products
// are exact in fp32.  Warp 0: TMA; warp 1: TMEM + MMA; warps 2-5: epilogue.
constexpr int kRWarps = 6;
constexpr int kRStages = 4;

__global__ void __launch_bounds__(kRWarps * 32, 1) router_gemm_kernel(
    const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x, const float* __restrict__ bias,
    int T, int E, int H, float* __restrict__ logits, int* status) {
  extern __shared__ __align__(1024) unsigned char rsm_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(rsm_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sA = base;                                  // kRStages x 16 KB
  unsigned char* sB = sA + kRStages * kAStageBytes;          // kRStages x 16 KB
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kRStages * kBStageBytes);
  uint64_t* empty = full + kRStages;
  uint64_t* acc_full = empty + kRStages;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kRStages; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&acc_full[i], 1); mbar_init(&acc_empty[i], 4); }
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();
  pdl_launch_dependents();
  const int mt = E / PBM, ntn = (T + PBN - 1) / PBN, ntiles = mt * ntn, KB = H / PBK;

  if (warp == 0 && lane == 0) {
    int kc = 0;
    for (int t = blockIdx.x; t < ntiles && !*abort_flag; t += gridDim.x) {
      const int m = t % mt, n = t / mt;
      for (int kb = 0; kb < KB; ++kb, ++kc) {
        const int s = kc % kRStages;
        if (kc >= kRStages && !mbar_wait(&empty[s], ((kc / kRStages) - 1) & 1, abort_flag)) {
          *abort_flag = 1; report_error(status, MOE_ERR_TIMEOUT, 30); break;
        }
        mbar_arrive_expect_tx(&full[s], kAStageBytes + kBStageBytes);
        tma_load_2d(sA + s * kAStageBytes, &tm_w, kb * PBK, m * PBM, &full[s]);
        tma_load_2d(sB + s * kBStageBytes, &tm_x, kb * PBK, n * PBN, &full[s]);
      }
    }
    for (int i = max(0, kc - kRStages); i < kc; ++i)
      if (!mbar_wait(&full[i % kRStages], (i / kRStages) & 1, nullptr)) report_error(status, MOE_ERR_TIMEOUT, 31);
  } else if (warp == 1 && lane == 0) {
    int kc = 0, tc = 0;
    for (int t = blockIdx.x; t < ntiles && !*abort_flag; t += gridDim.x, ++tc) {
      const int n = t / mt;
      const int buf = tc & 1;
      if (tc >= 2 && !mbar_wait(&acc_empty[buf], ((tc >> 1) - 1) & 1, abort_flag)) {
        *abort_flag = 1; report_error(status, MOE_ERR_TIMEOUT, 32); break;
      }
      tc_fence_after();
      const int nvalid = min(PBN, T - n * PBN);
      const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(((nvalid + 15) & ~15) >> 3) << 17) |
                             (uint32_t(PBM >> 4) << 24);   // D fp32, A/B bf16, K-major
      bool ok = true;
      for (int kb = 0; kb < KB; ++kb, ++kc) {
        const int s = kc % kRStages;
        if (!mbar_wait(&full[s], (kc / kRStages) & 1, abort_flag)) {
          *abort_flag = 1; report_error(status, MOE_ERR_TIMEOUT, 33); ok = false; break;
        }
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA + s * kAStageBytes), b0 = smem_u32(sB + s * kBStageBytes);
#pragma unroll
        for (int k = 0; k < PBK / 16; ++k)
          tc_mma(tmem_base + uint32_t(buf * PBN), sw128_desc(a0 + k * 32), sw128_desc(b0 + k * 32), idesc,
                 (kb | k) ? 1u : 0u);
        tc_commit(&empty[s]);
      }
      if (!ok) break;
      tc_commit(&acc_full[buf]);
    }
    if (kc > 0 && !mbar_wait(&empty[(kc - 1) % kRStages], ((kc - 1) / kRStages) & 1, nullptr))
      report_error(status, MOE_ERR_TIMEOUT, 34);
  } else if (warp >= 2) {
    const int q = warp & 3;
    const int r = q * 32 + lane;
    int tc = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++tc) {
      const int m = t % mt, n = t / mt;
      const int buf = tc & 1;
      if (*abort_flag || !mbar_wait(&acc_full[buf], (tc >> 1) & 1, abort_flag)) {
        if (!*abort_flag) { *abort_flag = 1; report_error(status, MOE_ERR_TIMEOUT, 35); }
        break;
      }
      tc_fence_after();
      const int e = m * PBM + r;
      const float b = bias ? __ldg(bias + e) : 0.f;
      const int nvalid = min(PBN, T - n * PBN);
      for (int n0 = 0; n0 < nvalid; n0 += 16) {
        uint32_t v[16];
        tmem_ld16(tmem_base + (uint32_t(q * 32) << 16) + uint32_t(buf * PBN + n0), v);
#pragma unroll
        for (int c = 0; c < 16; ++c)
          if (n0 + c < nvalid) logits[size_t(n * PBN + n0 + c) * E + e] = __uint_as_float(v[c]) + b;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols) : "memory");
  }
}

// ------------------------------------------------------------------ host
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

bool make_map(CUtensorMap* m, CUtensorMapDataType dt, int elem_bytes, const void* base, uint64_t inner,
              uint64_t rows, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * elem_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MODE, int BITS>
cudaError_t launch_gemm(const PrefillArgs& pa, const uint8_t* codes, const uint16_t* scales, const uint8_t* sh_codes,
                        const uint16_t* sh_scales, int E, bool has_shared, const uint16_t* bmat, int P, int num_sms,
                        cudaStream_t s) {
  using Gm = PGeom<BITS>;
  CUtensorMap mc, ms, msc, mss, mb;
  const uint64_t rb = uint64_t(pa.K) * BITS / 8, spr = uint64_t(pa.K) / Gm::BLOCK;
  const CUtensorMapSwizzle cswz = BITS == 4 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  const CUtensorMapSwizzle sswz = BITS == 4 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_32B;
  bool ok = make_map(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, codes, rb, uint64_t(E) * pa.rows_pe, Gm::IB, PBM, cswz) &&
            make_map(&ms, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, scales, spr, uint64_t(E) * pa.rows_pe, Gm::SB / 2, PBM, sswz) &&
            make_map(&mb, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, bmat, uint64_t(pa.K), uint64_t(P), PBK, PBN,
                     CU_TENSOR_MAP_SWIZZLE_128B);
  if (has_shared) {
    ok = ok && make_map(&msc, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, sh_codes, rb, uint64_t(pa.rows_pe), Gm::IB, PBM, cswz) &&
         make_map(&mss, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, sh_scales, spr, uint64_t(pa.rows_pe), Gm::SB / 2, PBM, sswz);
  } else {
    msc = mc;
    mss = ms;
  }
  if (!ok) return cudaErrorInvalidValue;
  constexpr int RAW_STRIDE = (Gm::RAW_BYTES + 1023) / 1024 * 1024;
  const size_t smem = 1024 + PNK * kGBStageBytes + PNR * RAW_STRIDE + kBarBytes + size_t(4 * E + 5) * 4 + 16 +
                      size_t(kTileTab) * 16;
  auto kern = prefill_gemm_kernel<MODE, BITS>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  return launch_pdl(kern, dim3(num_sms), dim3(PEp<MODE>::kThreads), smem, s, pa, mc, ms, msc, mss, mb);
}

}  // namespace

unsigned long long* g_prefill_timing = nullptr;
void set_prefill_timing(unsigned long long* buf) { g_prefill_timing = buf; }

bool router_gemm_supported(const moe_config& c, int T) {
  return T > 64 && c.num_experts % PBM == 0 && c.hidden % PBK == 0 && encode_fn() != nullptr;
}

cudaError_t launch_router_gemm(const moe_config& c, const uint16_t* router_w, const float* bias, const uint16_t* x,
                               int T, float* logits, int* status, int num_sms, cudaStream_t s) {
  CUtensorMap mw, mx;
  if (!make_map(&mw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, router_w, uint64_t(c.hidden), uint64_t(c.num_experts), PBK,
                PBM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, uint64_t(c.hidden), uint64_t(T), PBK, PBN,
                CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const size_t smem = 1024 + kRStages * (kAStageBytes + kBStageBytes) + 256;
  cudaError_t err = cudaFuncSetAttribute(router_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const int tiles = (c.num_experts / PBM) * ((T + PBN - 1) / PBN);
  return launch_pdl(router_gemm_kernel, dim3(min(num_sms, tiles)), dim3(kRWarps * 32), smem, s, mw, mx, bias, T,
                    c.num_experts, c.hidden, logits, status);
}

bool prefill_supported(const moe_config& c) {
  const int H = c.hidden, I = c.inter;
  const int bs = c.block;
  if (c.scale_fmt != 0) return false;              // fp8 block scales: the stand-alone GEMV reads them
  // the dequantizer takes one scale per 32 (4-bit) or 16 (2-bit) elements of a
  // packed stage; 4-bit blocks of 128 run on the CUDA-core GEMV at every size
  if (bs != (c.bits == 4 ? 32 : 16)) return false;
  if (H % RAWK || I % RAWK) return false;
  if ((2 * I) % PBM || H % PBM) return false;
  if ((H / bs * 2) % 16 || (I / bs * 2) % 16) return false;      // TMA row strides
  return encode_fn() != nullptr;
}

cudaError_t launch_prefill_ffn(const LayerArgs& a) {
  const moe_config& c = a.cfg;
  const int H = c.hidden, I = c.inter, bits = c.bits;
  RouteView rv;
  rv.T = a.T; rv.k = c.top_k; rv.E = c.num_experts; rv.shared = c.shared_inter > 0 ? 1 : 0;
  rv.status = reinterpret_cast<const int*>(a.ws + a.L.status);
  rv.ulist = reinterpret_cast<const int*>(a.ws + a.L.ulist);
  rv.offsets = reinterpret_cast<const int*>(a.ws + a.L.offsets);
  rv.pairs = reinterpret_cast<const int*>(a.ws + a.L.pairs);
  rv.inv = reinterpret_cast<const int*>(a.ws + a.L.inv);
  rv.topk_w = reinterpret_cast<const float*>(a.ws + a.L.topk_w);
  rv.woff = nullptr;
  const int P = a.L.P;
  uint16_t* xs = reinterpret_cast<uint16_t*>(a.ws + a.L.xs);
  uint16_t* hs = reinterpret_cast<uint16_t*>(a.ws + a.L.h);
  float* xinv = reinterpret_cast<float*>(a.ws + a.L.xscale);
  const int gblocks = max(1, min(a.num_sms * 8, (a.T + 7) / 8));    // one warp per token
  const size_t gsmem = size_t(8) * H * 2;                              // one fp16 row per warp
  cudaError_t err = cudaFuncSetAttribute(bits == 4 ? gather_tokens_kernel<4> : gather_tokens_kernel<2>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(gsmem));
  if (err != cudaSuccess) return err;
  err = bits == 4
      ? launch_pdl(gather_tokens_kernel<4>, dim3(gblocks), dim3(256), gsmem, a.stream, a.x, rv, H, xs, xinv, a.gated)
      : launch_pdl(gather_tokens_kernel<2>, dim3(gblocks), dim3(256), gsmem, a.stream, a.x, rv, H, xs, xinv, a.gated);
  if (err != cudaSuccess) return err;

  PrefillArgs g{};
  g.K = H; g.rows_pe = 2 * I; g.out_cols = I; g.rv = rv;
  g.ntoff = reinterpret_cast<const int*>(a.ws + a.L.ntoff);
  g.hout = hs; g.yout = nullptr; g.xinv = xinv;
  g.status = reinterpret_cast<int*>(a.ws + a.L.status);
  g.timing = g_prefill_timing;
  g.gated = a.gated;
  g.half_levels = c.half_levels;
  const bool sh = c.shared_inter > 0;
  err = bits == 4 ? launch_gemm<0, 4>(g, a.w.gate_up_codes, a.w.gate_up_scales, a.w.shared_gate_up_codes,
                                      a.w.shared_gate_up_scales, c.num_experts, sh, xs, P, a.num_sms, a.stream)
                  : launch_gemm<0, 2>(g, a.w.gate_up_codes, a.w.gate_up_scales, a.w.shared_gate_up_codes,
                                      a.w.shared_gate_up_scales, c.num_experts, sh, xs, P, a.num_sms, a.stream);
  if (err != cudaSuccess) return err;

  PrefillArgs d = g;
  d.K = I; d.rows_pe = H; d.out_cols = H;
  d.hout = nullptr; d.yout = reinterpret_cast<uint16_t*>(a.ws + a.L.y);
  d.timing = g_prefill_timing ? g_prefill_timing + size_t(a.num_sms) * kPTime : nullptr;
  return bits == 4 ? launch_gemm<1, 4>(d, a.w.down_codes, a.w.down_scales, a.w.shared_down_codes,
                                       a.w.shared_down_scales, c.num_experts, sh, hs, P, a.num_sms, a.stream)
                   : launch_gemm<1, 2>(d, a.w.down_codes, a.w.down_scales, a.w.shared_down_codes,
                                       a.w.shared_down_scales, c.num_experts, sh, hs, P, a.num_sms, a.stream);
}

}  // namespace moe
