// Internal declarations shared by the kernels and the C-ABI layer of libmoe.so.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stddef.h>

#include "../../include/moe_capi.h"

namespace moe {

// ------------------------------------------------------------ workspace ---
// One call's scratch, carved from the caller's workspace.  Every region starts
// on a 256-byte boundary.  P = T*k (+ T when the shared expert is present)
// counts token-expert pairs; pair positions are expert-major (sorted), the
// shared expert's pairs come last at positions T*k + t.
enum StatusSlot {
  ST_ERROR = 0,      // first failed device check (0 = none)
  ST_ERROR_AUX = 1,  // detail of that check
  ST_UCOUNT = 2,     // number of distinct routed experts selected
  ST_PATH = 3,       // fused decode with a tensor-core alternative: 1 = the grouped tcgen05 kernels run this call
  ST_COST_F = 4,     // that choice's inputs: CUDA-core cost units (gate/up + down) of the batch,
  ST_COST_T = 5,     //   and tensor-core k-blocks (128 rows x 128 tokens x 128 deep) of the batch
  ST_GRID_COUNT = 32,  // fused decode: grid barrier arrivals (own 128-byte line)
  ST_GRID_GEN = 64,    // fused decode: grid barrier generation (own 128-byte line)
  ST_COUNT = 96
};

// Tokens per chunk of the parallel grouping used for large batches.
constexpr int kGroupChunk = 64;

struct Layout {
  size_t status, logits, topk_idx, topk_w, counts, offsets, pairs, inv, ulist, woff_gu, woff_dn, ntoff, xhat, h,
      y, xs, xscale, chunk_hist, chunk_mask, gdone, total;
  int P;
};

__host__ __device__ inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

inline Layout make_layout(const moe_config& c, int T) {
  Layout L{};
  const int S = c.shared_inter > 0 ? 1 : 0;
  const int P = T * c.top_k + S * T;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align256(o + bytes); return at; };
  L.status = take(ST_COUNT * 4);
  L.logits = take(size_t(T) * c.num_experts * 4);
  L.topk_idx = take(size_t(T) * c.top_k * 4);
  L.topk_w = take(size_t(T) * c.top_k * 4);
  L.counts = take(size_t(c.num_experts) * 4);
  L.offsets = take(size_t(c.num_experts + 1) * 4);
  L.pairs = take(size_t(T) * c.top_k * 4);
  L.inv = take(size_t(T) * c.top_k * 4);
  L.ulist = take(size_t(c.num_experts + 1) * 4);
  L.woff_gu = take(size_t(c.num_experts + 2) * 4);
  L.woff_dn = take(size_t(c.num_experts + 2) * 4);
  L.ntoff = take(size_t(c.num_experts + 2) * 4);
  L.xhat = take(size_t(T) * c.hidden * 2);
  L.h = take(size_t(P) * c.inter * 4);
  L.y = take(size_t(P) * c.hidden * 4);
  L.xs = take(size_t(P) * c.hidden * 2);
  L.xscale = take(size_t(P) * 4);
  L.chunk_hist = take(size_t((T + kGroupChunk - 1) / kGroupChunk) * c.num_experts * 4);
  L.chunk_mask = take(size_t((T + kGroupChunk - 1) / kGroupChunk) * 2 * c.num_experts * 4);   // 64-token chunks
  L.gdone = take(size_t(c.num_experts + 2) * 4);   // fused decode: gate/up stages finished per slot
  L.total = o;
  L.P = P;
  return L;
}

// Everything a kernel of the layer needs to find the routing results.
struct RouteView {
  int T, k, E, shared;              // shared: 1 when the shared expert exists
  const int* status;                // [ST_COUNT]
  const int* ulist;                 // [E+1] touched experts ascending, E = shared
  const int* offsets;               // [E+1]
  const int* pairs;                 // [T*k] pair id t*k+j at each routed position
  const int* inv;                   // [T*k] position of pair t*k+j
  const float* topk_w;              // [T*k]
  const int* woff;                  // [nslots+1] work-unit prefix of one GEMV pass
};

// Token range of a slot of the touched-expert list: a routed expert e -> its
// sorted positions; the shared expert (id E) -> positions T*k .. T*k+T-1.
__device__ __forceinline__ void slot_range(const RouteView& rv, int slot, int* e_out, int* p0, int* n) {
  const int e = __ldcg(rv.ulist + slot);
  *e_out = e;
  if (e >= rv.E) {
    *p0 = rv.T * rv.k;
    *n = rv.T;
  } else {
    *p0 = __ldcg(rv.offsets + e);
    *n = __ldcg(rv.offsets + e + 1) - *p0;
  }
}

// Tokens per tensor-core tile of the prefill path.
constexpr int kPrefillTileN = 128;

// Work decomposition of one decode GEMV pass, shared by the grouping kernel
// (which writes the per-slot work prefix) and the GEMV kernel.
struct PassPlan {
  int ntc;    // tokens staged per chunk
  int spe;    // stages (row groups) per expert
};
// Work of one stage in balancing units, so that CTAs get equal time, not
// only equal bytes.  A stage's tokens are multiplied in groups of at most 4
// (1, 2 or 4 token slots, a group of 3 runs as 4); each group pays about
// 4 units for decoding the stage's codes and 3 per token slot.
__host__ __device__ inline int stage_cost(int tokens) {
  const int full = tokens >> 2, rest = tokens & 3;
  return full * (4 + 4 * 3) + (rest == 0 ? 0 : rest == 1 ? 4 + 3 : rest == 2 ? 4 + 2 * 3 : 4 + 4 * 3);
}
// Work of one expert slot of n tokens in a pass: its chunks of at most ntc
// tokens, each over the pass's spe stages.
__host__ __device__ inline int pass_cost(const PassPlan& pp, int n) {
  const int full = n / pp.ntc, rest = n % pp.ntc;
  return pp.spe * (full * stage_cost(pp.ntc) + (rest ? stage_cost(rest) : 0));
}

// -------------------------------------------------------------- device ---
__device__ __forceinline__ void pdl_wait() {
#if defined(__CUDA_ARCH__) && __CUDA_ARCH__ >= 900
  asm volatile("griddepcontrol.wait;" ::: "memory");
#endif
}
__device__ __forceinline__ void pdl_launch_dependents() {
#if defined(__CUDA_ARCH__) && __CUDA_ARCH__ >= 900
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
#endif
}

// Streaming 16-byte load of read-once weight bytes: read-only path, no L1 allocation.
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}
__device__ __forceinline__ uint32_t ld_stream4(const void* p) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ uint2 ld_stream8(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}
__device__ __forceinline__ uint16_t ld_stream2(const void* p) {
  uint16_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}

// ------------------------------------------------ mbarrier / bulk copy ---
// Every wait is bounded: after kWaitLimitCycles SM clock cycles (1-3 s at the
// B200's clocks; the SM cycle counter is read, as it costs a few cycles where
// %globaltimer costs tens of nanoseconds inside a spin) or when the CTA's
// abort flag is raised it gives up and returns false; the caller records
// MOE_ERR_TIMEOUT in the status word and skips the remaining work.
constexpr long long kWaitLimitCycles = 3000000000ll;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Waits for the phase of `bar` with the given parity; false on timeout/abort.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (abort_flag && *abort_flag) return false;
    if (clock64() - t0 > kWaitLimitCycles) return false;
  }
}
// 1-D TMA: `bytes` (multiple of 16, both addresses 16-byte aligned) from
// global to this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
// L2 policy for bytes read exactly once (the expert weights of a decode
// step): evicted first, so the stream does not push the kernel's code, the
// tokens and the routing scratch out of L2.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
// bulk_g2s with an L2 cache policy.
__device__ __forceinline__ void bulk_g2s_hint(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                              uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
      ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
// Records the first failure in the status word (0 = none).
__device__ __forceinline__ void report_error(int* status, int code, int aux) {
  if (atomicCAS(status, 0, code) == 0) atomicExch(status + 1, aux);
}

// (a & b) ^ c in one instruction.
__device__ __forceinline__ uint32_t lop_and_xor(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
// (a & b) | c in one instruction.
__device__ __forceinline__ uint32_t lop_and_or(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// ---------------------------------------------------------------- top-k ---
// Unsigned key with the order of the float (for non-NaN values); 0 is below
// every real key and marks a taken or absent logit.
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Largest of a lane's NPL keys and its slot, the lower slot on equal keys
// (a balanced tree, so the dependency chain is log2(NPL) deep).
template <int NPL>
__device__ __forceinline__ void lane_best(const uint32_t (&key)[NPL], uint32_t& bk, int& bm) {
  uint32_t kk[NPL];
  int mm[NPL];
#pragma unroll
  for (int m = 0; m < NPL; ++m) { kk[m] = key[m]; mm[m] = m; }
#pragma unroll
  for (int w = 1; w < NPL; w <<= 1)
#pragma unroll
    for (int m = 0; m + w < NPL; m += 2 * w)
      if (kk[m + w] > kk[m]) { kk[m] = kk[m + w]; mm[m] = mm[m + w]; }
  bk = kk[0];
  bm = mm[0];
}

// Top-k of one token's E logits by one warp: the k largest in descending
// order, equal logits by ascending expert id, then their softmax weights
// renormalised over the selection (the softmax maximum is the first pick).
// Lane l holds experts l, l+32, ...  The k-th largest of the 32 lane maxima,
// theta, bounds the selection from below (those k lanes already hold k values
// >= theta), so only the logits >= theta are candidates; when there are at
// most 32 of them they are ranked all at once through `scratch` (32 uint2 of
// shared memory for this warp), otherwise k rounds of warp maxima decide.
// CG reads the logits around L1 (they were written by other CTAs of the same
// launch).  Optionally marks the token in the picked experts' token masks
// (shared memory, word tmask[(t / 32) * E + expert], bit t % 32).
template <int NPL, bool CG>
__device__ __forceinline__ void warp_topk(const float* lrow, int k, int E, int* idx_out, float* w_out,
                                          uint2* scratch, unsigned* tmask = nullptr, int t = 0) {
  const int lane = threadIdx.x & 31;
  uint32_t key[NPL];
#pragma unroll
  for (int m = 0; m < NPL; ++m) {
    const int e = lane + 32 * m;
    key[m] = e < E ? order_key(CG ? __ldcg(lrow + e) : lrow[e]) : 0u;
  }
  uint32_t lb = key[0];
#pragma unroll
  for (int m = 1; m < NPL; ++m) lb = max(lb, key[m]);
  int r = 0;                       // rank of this lane's maximum among the 32
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const uint32_t o = __shfl_sync(0xffffffffu, lb, j);
    r += (o > lb) || (o == lb && j < lane);
  }
  const unsigned sel = __ballot_sync(0xffffffffu, r == k - 1);
  const uint32_t theta = __shfl_sync(0xffffffffu, lb, __ffs(sel) - 1);
  int nc = 0;
#pragma unroll
  for (int m = 0; m < NPL; ++m) nc += key[m] >= theta ? 1 : 0;
  int inc = nc;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  const int C = __shfl_sync(0xffffffffu, inc, 31);
  uint32_t my_key = 0;
  int my_idx = 0;
  if (C <= 32) {
    int w = inc - nc;
#pragma unroll
    for (int m = 0; m < NPL; ++m)
      if (key[m] >= theta) scratch[w++] = make_uint2(key[m], uint32_t(lane + 32 * m));
    __syncwarp();
    uint32_t ck = 0, ce = 0;
    int rank = 32;
    if (lane < C) {
      const uint2 cc = scratch[lane];
      ck = cc.x;
      ce = cc.y;
      rank = 0;
      for (int j = 0; j < C; ++j) {
        const uint2 o = scratch[j];
        rank += (o.x > ck) || (o.x == ck && o.y < ce);
      }
    }
    __syncwarp();
    if (rank < k) scratch[rank] = make_uint2(ck, ce);
    __syncwarp();
    if (lane < k) {
      const uint2 cc = scratch[lane];
      my_key = cc.x;
      my_idx = int(cc.y);
    }
    __syncwarp();
  } else {
    uint32_t bk;
    int bm;
    lane_best<NPL>(key, bk, bm);
    for (int j = 0; j < k; ++j) {
      const uint32_t mx = __reduce_max_sync(0xffffffffu, bk);
      const uint32_t we = __reduce_min_sync(0xffffffffu, bk == mx ? uint32_t(lane + 32 * bm) : 0xffffffffu);
      if (lane == j) { my_key = mx; my_idx = int(we); }
      if (int(we & 31u) == lane) {
#pragma unroll
        for (int m = 0; m < NPL; ++m)
          if (m == bm) key[m] = 0u;
        lane_best<NPL>(key, bk, bm);
      }
    }
  }
  const float my_logit = key_value(my_key);
  const float top = __shfl_sync(0xffffffffu, my_logit, 0);
  const float ex = lane < k ? expf(my_logit - top) : 0.f;
  float sum = ex;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane < k) {
    idx_out[lane] = my_idx;
    w_out[lane] = ex / sum;
    if (tmask) atomicOr(&tmask[(t >> 5) * E + my_idx], 1u << (t & 31));
  }
}

__device__ __forceinline__ __half2 u32_as_h2(uint32_t v) { return *reinterpret_cast<__half2*>(&v); }
__device__ __forceinline__ uint32_t h2_as_u32(__half2 v) { return *reinterpret_cast<uint32_t*>(&v); }

// In-register decode of packed codes to signed integers q = c - 2^(bits-1),
// exact in fp16.  A 16-bit lane of the form 0x6400 | (c << n) is the fp16
// number 1024 + c * 2^n; one fused multiply-add by 2^-n and -(1024/2^n +
// offset) leaves q.  Each half2 carries two elements that sit 16 bits apart in
// the source word, so the activation vector is stored in the matching order.
//
// 4-bit, one 32-bit word = 8 elements e0..e7 (e_j at bits 4j):
//   out[0] = (q0, q4)  out[1] = (q1, q5)  out[2] = (q2, q6)  out[3] = (q3, q7)
__device__ __forceinline__ void decode_q4x8(uint32_t v, __half2 out[4]) {
  const uint32_t MAGIC = 0x64006400u;
  const uint32_t lo0 = lop_and_or(v, 0x000F000Fu, MAGIC);
  const uint32_t hi0 = lop_and_or(v, 0x00F000F0u, MAGIC);
  const uint32_t v8 = v >> 8;
  const uint32_t lo1 = lop_and_or(v8, 0x000F000Fu, MAGIC);
  const uint32_t hi1 = lop_and_or(v8, 0x00F000F0u, MAGIC);
  const __half2 sub_lo = u32_as_h2(0x64086408u);          // 1032 = 1024 + 8
  const __half2 mul_hi = u32_as_h2(0x2C002C00u);          // 1/16
  const __half2 add_hi = u32_as_h2(0xD480D480u);          // -72 = -(64 + 8)
  out[0] = __hsub2(u32_as_h2(lo0), sub_lo);
  out[1] = __hfma2(u32_as_h2(hi0), mul_hi, add_hi);
  out[2] = __hsub2(u32_as_h2(lo1), sub_lo);
  out[3] = __hfma2(u32_as_h2(hi1), mul_hi, add_hi);
}

// Half-integer levels, q = c - 7.5: every field is first placed four bits up
// (0x6400 | (c << 4) = 1024 + 16 c), so one fused multiply-add by 1/16 and
// -71.5 leaves q; same pair order as decode_q4x8.
__device__ __forceinline__ void decode_q4x8_half(uint32_t v, __half2 out[4]) {
  const uint32_t MAGIC = 0x64006400u;
  const __half2 mul = u32_as_h2(0x2C002C00u);             // 1/16
  const __half2 add = u32_as_h2(0xD478D478u);             // -71.5 = -(64 + 7.5)
  out[0] = __hfma2(u32_as_h2(lop_and_or(v << 4, 0x00F000F0u, MAGIC)), mul, add);
  out[1] = __hfma2(u32_as_h2(lop_and_or(v, 0x00F000F0u, MAGIC)), mul, add);
  out[2] = __hfma2(u32_as_h2(lop_and_or(v >> 4, 0x00F000F0u, MAGIC)), mul, add);
  out[3] = __hfma2(u32_as_h2(lop_and_or(v >> 8, 0x00F000F0u, MAGIC)), mul, add);
}

// 2-bit, one 32-bit word = 16 elements e0..e15 (e_j at bits 2j):
//   out[j] = (q_j, q_{j+8}) for j = 0..7
__device__ __forceinline__ void decode_q2x16(uint32_t v, __half2 out[8]) {
  const uint32_t MAGIC = 0x64006400u;
  const __half2 sub1 = u32_as_h2(0x64026402u);            // 1026 = 1024 + 2
  const __half2 m4 = u32_as_h2(0x34003400u), a4 = u32_as_h2(0xDC08DC08u);    // 1/4,  -258
  const __half2 m16 = u32_as_h2(0x2C002C00u), a16 = u32_as_h2(0xD420D420u);  // 1/16, -66
  const __half2 m64 = u32_as_h2(0x24002400u), a64 = u32_as_h2(0xCC80CC80u);  // 1/64, -18
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const uint32_t w = half ? (v >> 8) : v;
    out[4 * half + 0] = __hsub2(u32_as_h2(lop_and_or(w, 0x00030003u, MAGIC)), sub1);
    out[4 * half + 1] = __hfma2(u32_as_h2(lop_and_or(w, 0x000C000Cu, MAGIC)), m4, a4);
    out[4 * half + 2] = __hfma2(u32_as_h2(lop_and_or(w, 0x00300030u, MAGIC)), m16, a16);
    out[4 * half + 3] = __hfma2(u32_as_h2(lop_and_or(w, 0x00C000C0u, MAGIC)), m64, a64);
  }
}
// Half-integer levels, q = c - 1.5 (four levels +-0.5, +-1.5): the lowest
// field is moved up two bits first so that every offset 1024 / 2^n + 1.5 is
// exact in fp16; same pair order as decode_q2x16.
__device__ __forceinline__ void decode_q2x16_half(uint32_t v, __half2 out[8]) {
  const uint32_t MAGIC = 0x64006400u;
  const __half2 m4 = u32_as_h2(0x34003400u), a4 = u32_as_h2(0xDC06DC06u);    // 1/4,  -257.5
  const __half2 m16 = u32_as_h2(0x2C002C00u), a16 = u32_as_h2(0xD418D418u);  // 1/16, -65.5
  const __half2 m64 = u32_as_h2(0x24002400u), a64 = u32_as_h2(0xCC60CC60u);  // 1/64, -17.5
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const uint32_t w = half ? (v >> 8) : v;
    out[4 * half + 0] = __hfma2(u32_as_h2(lop_and_or(w << 2, 0x000C000Cu, MAGIC)), m4, a4);
    out[4 * half + 1] = __hfma2(u32_as_h2(lop_and_or(w, 0x000C000Cu, MAGIC)), m4, a4);
    out[4 * half + 2] = __hfma2(u32_as_h2(lop_and_or(w, 0x00300030u, MAGIC)), m16, a16);
    out[4 * half + 3] = __hfma2(u32_as_h2(lop_and_or(w, 0x00C000C0u, MAGIC)), m64, a64);
  }
}

// Eight fp32 values rounded to bf16 (round to nearest even) as one 16-byte
// word group, element 2i in the low half of word i; in registers.
__device__ __forceinline__ uint4 pack_bf16x8(const float (&a)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 b = __floats2bfloat162_rn(a[2 * i], a[2 * i + 1]);
    w[i] = *reinterpret_cast<const uint32_t*>(&b);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Packs G fp32 values of one code group (k order), times mul, into the fp16
// pair order of the integer decoders -- word w = (v[w], v[w + G/2]), i.e. the
// element at position decode_slot(j) -- as G/8 16-byte parts, in registers
// (no local array, one paired conversion per word).
template <int G>
__device__ __forceinline__ void pack_pair_order(const float (&v)[G], float mul, uint4 (&parts)[G / 8]) {
  constexpr int HALF = G / 2;
  uint32_t w[HALF];
#pragma unroll
  for (int i = 0; i < HALF; ++i) {
    const __half2 h = __floats2half2_rn(v[i] * mul, v[i + HALF] * mul);
    w[i] = *reinterpret_cast<const uint32_t*>(&h);
  }
#pragma unroll
  for (int q = 0; q < G / 8; ++q) parts[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
}

// Position, inside a group of 8 (4-bit) or 16 (2-bit) consecutive elements,
// of element j in the half2 order produced by the decoders above.
__host__ __device__ inline int decode_slot(int bits, int j) {
  return bits == 4 ? (j & 3) * 2 + (j >> 2) : (j & 7) * 2 + (j >> 3);
}

// ------------------------------------------------------------- launches ---
struct LayerArgs {
  moe_config cfg;
  moe_layer_weights w;
  int T;
  const uint16_t* x;       // [T][H] bf16 layer input (post-norm when stacked)
  uint16_t* y;             // [T][H] bf16 output (layer) or the residual stream (stack)
  bool residual;           // y <- bf16(y + out) and refresh xhat for the next layer
  uint16_t* xhat_next;     // stack: normalised input of the next layer (or nullptr)
  char* ws;
  Layout L;
  int num_sms;
  cudaStream_t stream;
  int gated = 0;                  // run the tensor-core kernels only if the fused decode kernel handed over
  int ep_rank = 0, ep_size = 1;   // expert-parallel share: experts e with e % ep_size == ep_rank
  float* y_f32 = nullptr;         // [T][H] fp32 partial output (expert-parallel share) instead of y
  int y_half = 0;                 // the per-pair rows Y are fp16 (tensor-core path), else fp32
};

cudaError_t launch_rmsnorm(const uint16_t* x, uint16_t* xhat, int T, int H, cudaStream_t s);
cudaError_t launch_route(const moe_config& c, const uint16_t* router_w, const float* bias,
                         const uint16_t* x, int T, char* ws, const Layout& L, int num_sms,
                         cudaStream_t s);
cudaError_t launch_decode_ffn(const LayerArgs& a, cudaEvent_t between = nullptr);
void decode_plans(const moe_config& c, PassPlan* gu, PassPlan* dn);
cudaError_t launch_combine(const LayerArgs& a);
cudaError_t launch_prefill_ffn(const LayerArgs& a);
bool fused_supported(const moe_config& c, int T);
void set_fused_timing(unsigned long long* buf);
void set_prefill_timing(unsigned long long* buf);
extern unsigned long long* g_prefill_timing;
cudaError_t launch_status_reset(int* status, cudaStream_t s);
cudaError_t launch_fused_decode(const moe_config& c, const moe_layer_weights* layers, int L, const uint16_t* x,
                                uint16_t* y, bool stack, int T, int* trace, char* ws, const Layout& Lw, int num_sms,
                                cudaStream_t s, int hybrid = 0);
bool prefill_supported(const moe_config& c);
// The argument checks of moe_layer_forward short of the workspace (MOE_OK for
// T == 0, which is a no-op).
int check_layer_args(const moe_config* cfg, const moe_layer_weights* w, const uint16_t* x, int32_t T,
                     const uint16_t* y);
// Decode-path choice for single layers of 32..64 tokens: 0 = by the cost
// model after routing, 1 = always the fused CUDA-core kernel, 2 = always the
// grouped tensor-core kernels (measurement hook moe_debug_decode_path).
void set_decode_path_mode(int mode);
int decode_path_mode();
bool router_gemm_supported(const moe_config& c, int T);
cudaError_t launch_router_gemm(const moe_config& c, const uint16_t* router_w, const float* bias, const uint16_t* x,
                               int T, float* logits, int* status, int num_sms, cudaStream_t s);
cudaError_t launch_dequant_rows(int bits, int block, int half_levels, int scale_fmt, const uint8_t* codes,
                                const void* scales, const float* row_scales,
                                int row0, int rows, int cols, float* out, cudaStream_t s);
bool decode_shape_supported(int bits, int H, int I);

// Launch helper: programmatic dependent launch (the kernel may start while
// the previous kernel on the stream drains; it calls pdl_wait() before
// reading that kernel's results).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace moe
