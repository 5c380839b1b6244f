// Router logits, top-k selection with renormalised gates, and the counting
// sort that turns the selection into per-expert token lists.
//
// The router is the light gating network that picks the Top-K experts per
// token ("Running a 125B Model on a Single RTX 5090: Strata Benchmarks Qwen3.8
// Flash Next", section "Layer 1: On-Demand MoE Expert Scheduling"); per layer
// the GPU works out which 10 of 512 experts each token needs ("Strata Open
// Source Project: Run a 125B Model Locally on a Home PC", section "The
// 'Doorbell' Mechanism").  Gates: softmax over the selected logits (the full
// softmax renormalised over the selection); ties go to the smaller expert.
#include "moe_internal.cuh"

namespace moe {

namespace {

constexpr int kRouterWarps = 4;        // experts per router CTA (one warp each)
constexpr int kRouterTokTile = 16;     // tokens staged in shared memory at a time
constexpr int kRouterTokBlock = 256;   // tokens per CTA along grid.y
constexpr int kGroupThreads = 1024;    // the single grouping CTA

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(uint32_t(b) << 16);
}

// ------------------------------------------------------------------ rmsnorm
// xhat[t] = bf16(x[t] / sqrt(mean(x[t]^2) + 1e-6)), one CTA of 256 threads per
// token.  The sum of squares runs in the same order as the norm that
// combine_kernel fuses into the residual add (each thread 8 consecutive
// elements per step of 2048, then the warps in order), so a layer gets the
// same normalised input whichever of the two computed it.
__global__ void __launch_bounds__(256) rmsnorm_kernel(const uint16_t* __restrict__ x,
                                                      uint16_t* __restrict__ xhat, int H) {
  pdl_wait();
  const int t = blockIdx.x;
  const uint16_t* row = x + size_t(t) * H;
  float ss = 0.f;
  for (int h0 = threadIdx.x * 8; h0 < H; h0 += 256 * 8) {
    const uint4 xv = *reinterpret_cast<const uint4*>(row + h0);
    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float lo = __uint_as_float(xw[i] << 16), hi = __uint_as_float(xw[i] & 0xFFFF0000u);
      ss = fmaf(lo, lo, ss);
      ss = fmaf(hi, hi, ss);
    }
  }
  __shared__ float red[8];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
  for (int i = 0; i < (int)(blockDim.x >> 5); ++i) tot += red[i];
  const float r = 1.0f / sqrtf(tot / float(H) + 1e-6f);
  pdl_launch_dependents();
  for (int h = threadIdx.x; h < H; h += blockDim.x) {
    const __nv_bfloat16 o = __float2bfloat16_rn(bf16_bits_to_float(row[h]) * r);
    xhat[size_t(t) * H + h] = *reinterpret_cast<const uint16_t*>(&o);
  }
}

// ---------------------------------------------------------- router logits
// logits[t][e] = sum_h x[t][h] * Wr[e][h] (+ bias[e]) in fp32.  Each warp owns
// one expert row; its lanes read 16-byte pieces of the row (a warp load is
// 512 contiguous bytes) and the row stays in registers while the warp walks
// the tokens, which are staged in shared memory kRouterTokTile at a time.
template <int H>
__global__ void __launch_bounds__(kRouterWarps * 32) router_logits_kernel(
    const uint16_t* __restrict__ wr, const float* __restrict__ bias,
    const uint16_t* __restrict__ x, int T, int E, int tokens_per_cta, float* __restrict__ logits) {
  constexpr int PER_LANE = H / 256;   // 16-byte pieces per lane
  extern __shared__ __align__(16) uint16_t xs[];   // [kRouterTokTile][H]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * kRouterWarps + warp;
  uint4 wv[PER_LANE];
  if (e < E) {
    const uint16_t* row = wr + size_t(e) * H;
#pragma unroll
    for (int p = 0; p < PER_LANE; ++p) wv[p] = ld_stream16(row + (p * 32 + lane) * 8);
  }
  const float b = (e < E && bias) ? bias[e] : 0.f;
  pdl_wait();   // x may be produced by the previous kernel
  pdl_launch_dependents();
  const int t_lo = blockIdx.y * tokens_per_cta, t_hi = min(T, t_lo + tokens_per_cta);
  for (int t0 = t_lo; t0 < t_hi; t0 += kRouterTokTile) {
    const int nt = min(kRouterTokTile, t_hi - t0);
    __syncthreads();
    // stage nt token rows; loads are issued in batches of 8 per thread
    const int n16 = nt * H / 8;
    const uint4* src = reinterpret_cast<const uint4*>(x + size_t(t0) * H);
    for (int base = threadIdx.x; base < n16; base += kRouterWarps * 32 * 8) {
      uint4 v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int i = base + j * kRouterWarps * 32;
        if (i < n16) v[j] = __ldg(src + i);
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int i = base + j * kRouterWarps * 32;
        if (i < n16) reinterpret_cast<uint4*>(xs)[i] = v[j];
      }
    }
    __syncthreads();
    if (e < E) {
      for (int t = 0; t < nt; ++t) {
        float acc = 0.f;
#pragma unroll
        for (int p = 0; p < PER_LANE; ++p) {
          const uint4 xv = reinterpret_cast<const uint4*>(xs + t * H)[p * 32 + lane];
          const uint32_t wa[4] = {wv[p].x, wv[p].y, wv[p].z, wv[p].w};
          const uint32_t xa[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            acc = fmaf(__uint_as_float(wa[q] << 16), __uint_as_float(xa[q] << 16), acc);
            acc = fmaf(__uint_as_float(wa[q] & 0xFFFF0000u), __uint_as_float(xa[q] & 0xFFFF0000u), acc);
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) logits[size_t(t0 + t) * E + e] = acc + b;
      }
    }
  }
}

// ------------------------------------------------------------------ top-k
// One warp selects the k largest of E logits: lane l holds experts l + 32m.
// Each round takes the warp-wide maximum (ties to the smaller expert), the
// owner marks it taken.  Gates are a softmax over the k selected logits.
template <int NPL>
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                   int* __restrict__ idx, float* __restrict__ w) {
  __shared__ uint2 scratch[8][32];
  pdl_wait();
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t < T)
    warp_topk<NPL, false>(logits + size_t(t) * E, k, E, idx + size_t(t) * k, w + size_t(t) * k, scratch[threadIdx.x >> 5]);
  pdl_launch_dependents();
}

// -------------------------------------------------------------- grouping
// Stable counting sort of the T*k (token, slot) pairs by expert, in one CTA of
// 32 warps.  Warp w owns a contiguous token range; per-warp histograms give
// each warp's starting rank inside every expert, then each warp walks its
// tokens in order, so positions are sorted by expert, then by token.  Also
// writes the ascending list of selected experts (the shared expert appended
// as id E) and, when `fused_topk`, runs the top-k itself first (decode).
template <int NPL>
__global__ void __launch_bounds__(kGroupThreads) group_kernel(
    const float* __restrict__ logits, int fused_topk, int* __restrict__ idx, float* __restrict__ w,
    int T, int E, int k, int shared, int* __restrict__ status, int* __restrict__ counts_out,
    int* __restrict__ offsets_out, int* __restrict__ pairs_out, int* __restrict__ inv_out,
    int* __restrict__ ulist_out, int* __restrict__ api_counts, int* __restrict__ api_offsets,
    int* __restrict__ api_pairs, PassPlan pg, PassPlan pd, int* __restrict__ woff_gu,
    int* __restrict__ woff_dn, int* __restrict__ ntoff, int ep_rank, int ep_size) {
  extern __shared__ int sm[];
  constexpr int NW = kGroupThreads / 32;
  int* hist = sm;                       // [NW][E]
  int* offs = sm + NW * E;              // [E+1]
  int* scan = offs + E + 1;             // [kGroupThreads] scan scratch
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();
  if (fused_topk) {
    __shared__ uint2 topk_scratch[kGroupThreads / 32][32];
    for (int t = warp; t < T; t += NW)
      warp_topk<NPL, false>(logits + size_t(t) * E, k, E, idx + size_t(t) * k, w + size_t(t) * k, topk_scratch[warp]);
    __syncthreads();
    __threadfence_block();
  }
  for (int i = threadIdx.x; i < NW * E; i += kGroupThreads) hist[i] = 0;
  __syncthreads();
  const int tpw = (T + NW - 1) / NW;
  const int t_begin = min(T, warp * tpw), t_end = min(T, t_begin + tpw);
  for (int p = t_begin * k + lane; p < t_end * k; p += 32) {
    const int e = idx[p];
    if (e < 0 || e >= E) {              // never produced by the selection above
      atomicCAS(status + ST_ERROR, 0, 1);
      continue;
    }
    if (e % ep_size != ep_rank) continue;   // expert of another rank
    atomicAdd(&hist[warp * E + e], 1);
  }
  __syncthreads();
  // per-expert exclusive prefix over warps; counts
  for (int e = threadIdx.x; e < E; e += kGroupThreads) {
    int run = 0;
    for (int ww = 0; ww < NW; ++ww) {
      const int c = hist[ww * E + e];
      hist[ww * E + e] = run;
      run += c;
    }
    offs[e] = run;                      // count for now
  }
  __syncthreads();
  // exclusive scan of counts -> offsets (E <= kGroupThreads)
  {
    const int e = threadIdx.x;
    const int c = e < E ? offs[e] : 0;
    int v = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += n;
    }
    if (lane == 31) scan[warp] = v;
    __syncthreads();
    if (warp == 0) {
      int s = scan[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += n;
      }
      scan[lane] = s;                   // inclusive over warps
    }
    __syncthreads();
    const int excl = v - c + (warp > 0 ? scan[warp - 1] : 0);
    __syncthreads();
    if (e < E) {
      counts_out[e] = c;
      offsets_out[e] = excl;
      if (api_counts) api_counts[e] = c;
      if (api_offsets) api_offsets[e] = excl;
      offs[e] = excl;
    }
    if (e == E - 1) {
      offsets_out[E] = excl + c;
      if (api_offsets) api_offsets[E] = excl + c;
      offs[E] = excl + c;
    }
    // touched-expert list: scan of flags
    __syncthreads();
    const int f = (e < E && c > 0) ? 1 : 0;
    int fv = f;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, fv, o);
      if (lane >= o) fv += n;
    }
    if (lane == 31) scan[warp] = fv;
    __syncthreads();
    if (warp == 0) {
      int s = scan[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += n;
      }
      scan[lane] = s;
    }
    __syncthreads();
    const int fpos = fv - f + (warp > 0 ? scan[warp - 1] : 0);
    if (f) ulist_out[fpos] = e;
    if (threadIdx.x == 0) {
      const int U = scan[NW - 1];
      status[ST_UCOUNT] = U;
      if (shared) ulist_out[U] = E;
    }
  }
  __syncthreads();
  // work prefix of the two GEMV passes over the slots (touched experts, then
  // the shared expert), in balancing cost units.
  if (warp == 0) {
    const int U = scan[NW - 1];
    const int nslots = U + shared;
    int run_g = 0, run_d = 0, run_t = 0;
    for (int base = 0; base < nslots; base += 32) {
      const int u = base + lane;
      int n = 0;
      if (u < U) {
        const int e = ulist_out[u];
        n = offs[e + 1] - offs[e];
      } else if (u < nslots) {
        n = T;
      }
      int g = u < nslots ? pass_cost(pg, n) : 0;
      int d = u < nslots ? pass_cost(pd, n) : 0;
      int nt = u < nslots ? (n + kPrefillTileN - 1) / kPrefillTileN : 0;   // token tiles (prefill)
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int ng = __shfl_up_sync(0xffffffffu, g, o);
        const int nd = __shfl_up_sync(0xffffffffu, d, o);
        const int nn = __shfl_up_sync(0xffffffffu, nt, o);
        if (lane >= o) { g += ng; d += nd; nt += nn; }
      }
      if (u < nslots) {
        woff_gu[u + 1] = run_g + g;
        woff_dn[u + 1] = run_d + d;
        ntoff[u + 1] = run_t + nt;
      }
      run_g += __shfl_sync(0xffffffffu, g, 31);
      run_d += __shfl_sync(0xffffffffu, d, 31);
      run_t += __shfl_sync(0xffffffffu, nt, 31);
    }
    if (lane == 0) {
      woff_gu[0] = 0;
      woff_dn[0] = 0;
      ntoff[0] = 0;
    }
  }
  // stable scatter: each warp walks its tokens in order
  for (int t = t_begin; t < t_end; ++t) {
    if (lane < k) {
      const int q = t * k + lane;
      const int e = idx[q];
      if (e >= 0 && e < E && e % ep_size == ep_rank) {
        const int pos = offs[e] + hist[warp * E + e];
        hist[warp * E + e] += 1;        // distinct experts within one token
        pairs_out[pos] = q;
        inv_out[q] = pos;
        if (api_pairs) api_pairs[pos] = q;
      } else {
        inv_out[q] = -1;                // not computed on this rank
      }
    }
    __syncwarp();
  }
  pdl_launch_dependents();
}

// ------------------------------------------------- parallel grouping (large T)
// The same stable counting sort as group_kernel, spread over CTAs: each
// chunk of kGroupChunk tokens counts its pairs per expert; one CTA turns the
// counts into per-chunk bases, offsets, the touched-expert list and the work
// prefixes; each chunk then writes its pairs in token order.
// Large batches: a stable counting sort over 64-token chunks, with the order
// inside a chunk taken from per-expert token masks (bit t of chunk expert e:
// token t of the chunk picked e).  chunk_mask_kernel builds a chunk's masks and
// its per-expert counts; chunk_scan_kernel turns the counts into per-chunk
// bases, offsets, the touched-expert list and the work prefixes; and
// chunk_place_kernel puts pair (t, j) of expert e at
//   offset(e) + base(chunk, e) + (tokens of the chunk before t that picked e),
// every pair independently.
__global__ void __launch_bounds__(256) chunk_mask_kernel(const int* __restrict__ idx, int T, int k, int E,
                                                         int* __restrict__ chunk_hist, unsigned* __restrict__ chunk_mask,
                                                         int* __restrict__ status, int ep_rank, int ep_size) {
  extern __shared__ unsigned msk[];                 // [2][E]
  pdl_wait();
  pdl_launch_dependents();
  for (int i = threadIdx.x; i < 2 * E; i += blockDim.x) msk[i] = 0u;
  __syncthreads();
  const int t0 = blockIdx.x * kGroupChunk, t1 = min(T, t0 + kGroupChunk);
  for (int q = t0 * k + threadIdx.x; q < t1 * k; q += blockDim.x) {
    const int e = idx[q];
    if (e < 0 || e >= E) { atomicCAS(status + ST_ERROR, 0, 2); continue; }
    const int tl = q / k - t0;
    atomicOr(&msk[(tl >> 5) * E + e], 1u << (tl & 31));
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const unsigned m0 = msk[e], m1 = msk[E + e];
    chunk_hist[size_t(blockIdx.x) * E + e] = (e % ep_size == ep_rank) ? __popc(m0) + __popc(m1) : 0;
    chunk_mask[size_t(blockIdx.x) * 2 * E + e] = m0;
    chunk_mask[size_t(blockIdx.x) * 2 * E + E + e] = m1;
  }
}

// Exclusive block-wide scan of NV values per thread (all kGroupThreads
// threads), with the totals; scr: 32 * NV ints of shared memory.
template <int NV>
__device__ __forceinline__ void block_scan_n(const int (&v)[NV], int (&excl)[NV], int (&tot)[NV], int* scr) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int x[NV];
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    x[j] = v[j];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, x[j], o);
      if (lane >= o) x[j] += n;
    }
  }
  if (lane == 31) {
#pragma unroll
    for (int j = 0; j < NV; ++j) scr[j * 32 + warp] = x[j];
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    int before = 0, all = 0;
#pragma unroll 8
    for (int w = 0; w < kGroupThreads / 32; ++w) {
      const int s = scr[j * 32 + w];
      before += w < warp ? s : 0;
      all += s;
    }
    excl[j] = before + x[j] - v[j];
    tot[j] = all;
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kGroupThreads) chunk_scan_kernel(
    int nchunks, int T, int E, int shared, int* __restrict__ chunk_hist, int* __restrict__ status,
    int* __restrict__ counts_out, int* __restrict__ offsets_out, int* __restrict__ ulist_out,
    int* __restrict__ api_counts, int* __restrict__ api_offsets, PassPlan pg, PassPlan pd,
    int* __restrict__ woff_gu, int* __restrict__ woff_dn, int* __restrict__ ntoff) {
  __shared__ int scr[32 * 3];
  __shared__ int cnt[1025];
  pdl_wait();
  pdl_launch_dependents();
  const int e = threadIdx.x;
  int c = 0;
  if (e < E) {
    // per-chunk base of expert e = exclusive prefix over chunks; the loads of
    // 32 chunks are in flight together
    int run = 0;
    for (int ch0 = 0; ch0 < nchunks; ch0 += 32) {
      int v[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = ch0 + j < nchunks ? __ldcg(chunk_hist + size_t(ch0 + j) * E + e) : 0;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (ch0 + j < nchunks) chunk_hist[size_t(ch0 + j) * E + e] = run;
        run += v[j];
      }
    }
    c = run;
  }
  const int in2[2] = {c, (e < E && c > 0) ? 1 : 0};
  int ex2[2], tot2[2];
  block_scan_n<2>(in2, ex2, tot2, scr);
  if (e < E) {
    counts_out[e] = c;
    offsets_out[e] = ex2[0];
    cnt[e] = c;
    if (api_counts) api_counts[e] = c;
    if (api_offsets) api_offsets[e] = ex2[0];
    if (c > 0) ulist_out[ex2[1]] = e;
  }
  const int U = tot2[1];
  if (threadIdx.x == 0) {
    offsets_out[E] = tot2[0];
    if (api_offsets) api_offsets[E] = tot2[0];
    status[ST_UCOUNT] = U;
    if (shared) ulist_out[U] = E;
  }
  __syncthreads();
  // work prefixes over the slots (touched experts ascending, the shared
  // expert last): slot u of thread u, and slot 1024 (E = 1024 with every
  // expert touched and a shared expert) on thread 0's second pass
  const int nslots = U + shared;
  for (int base = 0; base < nslots; base += kGroupThreads) {
    const int u = base + threadIdx.x;
    int n = 0;
    if (u < U) n = cnt[ulist_out[u]];
    else if (u < nslots) n = T;
    const int in3[3] = {u < nslots ? pass_cost(pg, n) : 0, u < nslots ? pass_cost(pd, n) : 0,
                        u < nslots ? (n + kPrefillTileN - 1) / kPrefillTileN : 0};
    int ex3[3], tot3[3];
    block_scan_n<3>(in3, ex3, tot3, scr);
    const int g0 = base ? woff_gu[base] : 0, d0 = base ? woff_dn[base] : 0, n0 = base ? ntoff[base] : 0;
    __syncthreads();
    if (u < nslots) {
      woff_gu[u + 1] = g0 + ex3[0] + in3[0];
      woff_dn[u + 1] = d0 + ex3[1] + in3[1];
      ntoff[u + 1] = n0 + ex3[2] + in3[2];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) { woff_gu[0] = 0; woff_dn[0] = 0; ntoff[0] = 0; }
}

__global__ void __launch_bounds__(256) chunk_place_kernel(const int* __restrict__ idx, int T, int k, int E,
                                                          const int* __restrict__ chunk_base,
                                                          const unsigned* __restrict__ chunk_mask,
                                                          const int* __restrict__ offsets, int* __restrict__ pairs,
                                                          int* __restrict__ inv, int* __restrict__ api_pairs,
                                                          int ep_rank, int ep_size) {
  extern __shared__ unsigned pl[];             // masks [2][E], then the bases [E]
  int* base = reinterpret_cast<int*>(pl + 2 * E);
  pdl_wait();
  pdl_launch_dependents();
  const int ch = blockIdx.x;
  for (int i = threadIdx.x; i < 2 * E; i += blockDim.x) pl[i] = __ldcg(chunk_mask + size_t(ch) * 2 * E + i);
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    base[e] = __ldcg(offsets + e) + __ldcg(chunk_base + size_t(ch) * E + e);
  __syncthreads();
  const int t0 = ch * kGroupChunk, t1 = min(T, t0 + kGroupChunk);
  for (int q = t0 * k + threadIdx.x; q < t1 * k; q += blockDim.x) {
    const int e = idx[q];
    if (e < 0 || e >= E || e % ep_size != ep_rank) {
      inv[q] = -1;                             // not computed on this rank
      continue;
    }
    const int tl = q / k - t0;
    const unsigned m0 = pl[e];
    const int r = tl < 32 ? __popc(m0 & ((1u << tl) - 1u))
                          : __popc(m0) + __popc(pl[E + e] & ((1u << (tl - 32)) - 1u));
    const int pos = base[e] + r;
    pairs[pos] = q;
    inv[q] = pos;
    if (api_pairs) api_pairs[pos] = q;
  }
}

template <int NPL>
cudaError_t launch_topk_group(const moe_config& c, int T, char* ws, const Layout& L, bool fused,
                              int* api_counts, int* api_offsets, int* api_pairs, int ep_rank, int ep_size,
                              cudaStream_t s) {
  const size_t smem = (size_t(32) * c.num_experts + c.num_experts + 1 + kGroupThreads) * sizeof(int);
  auto kern = group_kernel<NPL>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  PassPlan pg{1, 1}, pd{1, 1};
  decode_plans(c, &pg, &pd);
  float* logits = reinterpret_cast<float*>(ws + L.logits);
  int* idx = reinterpret_cast<int*>(ws + L.topk_idx);
  float* w = reinterpret_cast<float*>(ws + L.topk_w);
  if (!fused) {
    err = launch_pdl(topk_kernel<NPL>, dim3((T + 7) / 8), dim3(256), 0, s, logits, T, c.num_experts,
                     c.top_k, idx, w);
    if (err != cudaSuccess) return err;
    if (T > 4 * kGroupChunk) {
      // large batch: parallel stable counting sort
      const int nch = (T + kGroupChunk - 1) / kGroupChunk, E = c.num_experts;
      int* hist = reinterpret_cast<int*>(ws + L.chunk_hist);
      int* status = reinterpret_cast<int*>(ws + L.status);
      unsigned* masks = reinterpret_cast<unsigned*>(ws + L.chunk_mask);
      err = launch_pdl(chunk_mask_kernel, dim3(nch), dim3(256), size_t(2 * E) * 4, s, (const int*)idx, T, c.top_k,
                       E, hist, masks, status, ep_rank, ep_size);
      if (err != cudaSuccess) return err;
      err = launch_pdl(chunk_scan_kernel, dim3(1), dim3(kGroupThreads), 0, s, nch, T, E, c.shared_inter > 0 ? 1 : 0,
                       hist, status, reinterpret_cast<int*>(ws + L.counts), reinterpret_cast<int*>(ws + L.offsets),
                       reinterpret_cast<int*>(ws + L.ulist), api_counts, api_offsets, pg, pd,
                       reinterpret_cast<int*>(ws + L.woff_gu), reinterpret_cast<int*>(ws + L.woff_dn),
                       reinterpret_cast<int*>(ws + L.ntoff));
      if (err != cudaSuccess) return err;
      return launch_pdl(chunk_place_kernel, dim3(nch), dim3(256), size_t(3 * E) * 4, s, (const int*)idx, T,
                        c.top_k, E, (const int*)hist, (const unsigned*)masks, (const int*)(ws + L.offsets),
                        reinterpret_cast<int*>(ws + L.pairs), reinterpret_cast<int*>(ws + L.inv), api_pairs, ep_rank,
                        ep_size);
    }
  }
  return launch_pdl(kern, dim3(1), dim3(kGroupThreads), smem, s, logits, fused ? 1 : 0, idx, w, T,
                    c.num_experts, c.top_k, c.shared_inter > 0 ? 1 : 0,
                    reinterpret_cast<int*>(ws + L.status), reinterpret_cast<int*>(ws + L.counts),
                    reinterpret_cast<int*>(ws + L.offsets), reinterpret_cast<int*>(ws + L.pairs),
                    reinterpret_cast<int*>(ws + L.inv), reinterpret_cast<int*>(ws + L.ulist), api_counts,
                    api_offsets, api_pairs, pg, pd, reinterpret_cast<int*>(ws + L.woff_gu),
                    reinterpret_cast<int*>(ws + L.woff_dn), reinterpret_cast<int*>(ws + L.ntoff), ep_rank, ep_size);
}

}  // namespace

cudaError_t launch_rmsnorm(const uint16_t* x, uint16_t* xhat, int T, int H, cudaStream_t s) {
  return launch_pdl(rmsnorm_kernel, dim3(T), dim3(256), 0, s, x, xhat, H);
}

cudaError_t launch_router_logits(const moe_config& c, const uint16_t* router_w, const float* bias,
                                 const uint16_t* x, int T, float* logits, cudaStream_t s) {
  // decode batches: 4 tokens per CTA so each CTA stages little; prefill: 256
  const int tpc = T <= 64 ? 4 : kRouterTokBlock;
  const dim3 grid((c.num_experts + kRouterWarps - 1) / kRouterWarps, (T + tpc - 1) / tpc);
  const dim3 block(kRouterWarps * 32);
  const size_t smem = size_t(kRouterTokTile) * c.hidden * 2;
  void (*kern)(const uint16_t*, const float*, const uint16_t*, int, int, int, float*) = nullptr;
  switch (c.hidden) {
    case 256: kern = router_logits_kernel<256>; break;
    case 512: kern = router_logits_kernel<512>; break;
    case 1024: kern = router_logits_kernel<1024>; break;
    case 2048: kern = router_logits_kernel<2048>; break;
    case 4096: kern = router_logits_kernel<4096>; break;
    default: return cudaErrorInvalidValue;
  }
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  return launch_pdl(kern, grid, block, smem, s, router_w, bias, x, T, c.num_experts, tpc, logits);
}

cudaError_t launch_topk_group_any(const moe_config& c, int T, char* ws, const Layout& L, bool fused,
                                  int* api_counts, int* api_offsets, int* api_pairs, int ep_rank, int ep_size,
                                  cudaStream_t s) {
  switch (c.num_experts / 32) {
    case 1: return launch_topk_group<1>(c, T, ws, L, fused, api_counts, api_offsets, api_pairs, ep_rank, ep_size, s);
    case 2: return launch_topk_group<2>(c, T, ws, L, fused, api_counts, api_offsets, api_pairs, ep_rank, ep_size, s);
    case 4: return launch_topk_group<4>(c, T, ws, L, fused, api_counts, api_offsets, api_pairs, ep_rank, ep_size, s);
    case 8: return launch_topk_group<8>(c, T, ws, L, fused, api_counts, api_offsets, api_pairs, ep_rank, ep_size, s);
    case 16: return launch_topk_group<16>(c, T, ws, L, fused, api_counts, api_offsets, api_pairs, ep_rank, ep_size, s);
    case 32: return launch_topk_group<32>(c, T, ws, L, fused, api_counts, api_offsets, api_pairs, ep_rank, ep_size, s);
    default: return cudaErrorInvalidValue;
  }
}

// Clears the workspace's status words (error code, counts, grid-barrier words)
// before a single-launch decode kernel; it lets that kernel launch at once
// (programmatic dependency) and the kernel waits for its completion before it
// touches the workspace.
__global__ void status_reset_kernel(int* status) {
  pdl_launch_dependents();
  pdl_wait();                    // whatever ran before on the stream has completed
  for (int i = threadIdx.x; i < ST_COUNT; i += blockDim.x) status[i] = 0;
}

cudaError_t launch_status_reset(int* status, cudaStream_t s) {
  return launch_pdl(status_reset_kernel, dim3(1), dim3(128), 0, s, status);
}

cudaError_t launch_route_full(const moe_config& c, const uint16_t* router_w, const float* bias,
                              const uint16_t* x, int T, char* ws, const Layout& L, int* api_counts,
                              int* api_offsets, int* api_pairs, cudaStream_t s, int ep_rank, int ep_size) {
  int nsm = 148;
  {
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  }
  cudaError_t err = router_gemm_supported(c, T)
      ? launch_router_gemm(c, router_w, bias, x, T, reinterpret_cast<float*>(ws + L.logits),
                           reinterpret_cast<int*>(ws + L.status), nsm, s)
      : launch_router_logits(c, router_w, bias, x, T, reinterpret_cast<float*>(ws + L.logits), s);
  if (err != cudaSuccess) return err;
  const bool fused = T <= 64;
  return launch_topk_group_any(c, T, ws, L, fused, api_counts, api_offsets, api_pairs, ep_rank, ep_size, s);
}

cudaError_t launch_route(const moe_config& c, const uint16_t* router_w, const float* bias,
                         const uint16_t* x, int T, char* ws, const Layout& L, int, cudaStream_t s) {
  return launch_route_full(c, router_w, bias, x, T, ws, L, nullptr, nullptr, nullptr, s, 0, 1);
}

}  // namespace moe
