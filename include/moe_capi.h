/*
 * moe_capi.h -- C ABI of the routed, quantized-expert MoE FFN layer for B200
 * (sm_100a).  Library: libmoe.so (built in-tree into quantized_expert_ffn_moe_b200/).
 *
 * The operation.  The transformer block's FFN is replaced by many parallel
 * expert sub-networks plus a light gating network (router) that picks the
 * Top-K experts per token ("Running a 125B Model on a Single RTX 5090: Strata
 * Benchmarks Qwen3.8 Flash Next", section "Layer 1: On-Demand MoE Expert
 * Scheduling"); 512 experts per layer with 10 selected per token ("Strata Open
 * Source Project: Run a 125B Model Locally on a Home PC", section "How Strata
 * Makes Your Entire PC Work Together"); one shared expert is active for every
 * token besides the routed ones ("How a 125B Model Reaches 100 Tok/s on an RTX
 * 4090", section "The model is large on paper, sparse in practice"); expert
 * weights are symmetric, group-wise quantised 4-bit or 2-bit integers
 * ("Running Massive Language Models on Consumer Hardware Without Breaking the
 * Bank", section "Quantization Techniques That Actually Work").
 *
 * Per token x (bf16, hidden H):
 *   l_e   = sum_h x_h Wr[e,h] (+ b_e)                  fp32 accumulation
 *   S     = the k largest l_e, slots by descending logit, ties -> smaller e
 *   w_j   = softmax over the selected logits (= full softmax renormalised)
 *   FFN_e = W_down,e (silu(W_gate,e x) * (W_up,e x)),   W = q * scale (q from the code)
 *   out   = g(x) FFN_shared(x) + sum_j w_j FFN_{S_j}(x)  slot order, fp32, -> bf16
 *   g(x)  = 1, or sigmoid(sum_h x_h Wg[h]) when a shared-expert gate vector Wg is given
 *
 * Packed weight format (all arrays row-major, dense, caller-owned, device
 * memory, 16-byte aligned):
 *   codes : one byte holds 8/bits elements of a row; element j of a row is at
 *           byte j*bits/8, bit offset (j*bits)%8 (lower element in lower bits);
 *           stored code c = q + 2^(bits-1), q in [-(2^(bits-1)-1), 2^(bits-1)-1]
 *           (integer levels; 2-bit is then ternary), or, with half_levels,
 *           c = q + (2^bits - 1)/2, q in {-(2^(bits-1) - 1/2), ..., 2^(bits-1) - 1/2}
 *           (the 2^bits half-integer levels; 2-bit: +-1/2, +-3/2)
 *   scales: one IEEE fp16 per block of `block` consecutive elements of a row
 *   gate/up: one [2I, H] matrix per expert, row 2i = gate row i, row 2i+1 =
 *           up row i; down: [H, I] per expert.  Experts are stacked densely.
 * Supported: bits/block in {4/32, 2/16}; H % 256 == 0; I % 128 == 0;
 * 1 <= k <= 16, k <= E <= 1024; shared_inter in {0, inter}.
 *
 * Conventions.  All calls are asynchronous on `stream` (a cudaStream_t passed
 * as void*; NULL = legacy default stream) and never allocate or free device
 * memory: scratch comes from the caller's `workspace` (device, 256-byte
 * aligned, at least moe_workspace_bytes()).  Arguments are validated on the
 * host before any launch; on error nothing is launched and a negative
 * moe_status is returned.  T == 0 returns MOE_OK and launches nothing.  The
 * same inputs give bitwise identical outputs on every call (no float atomics).
 * Calls that share a workspace must not overlap in time on the device.
 */
#ifndef MOE_CAPI_H
#define MOE_CAPI_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = -1,   /* null/misaligned pointer, negative size         */
  MOE_ERR_UNSUPPORTED = -2,   /* shape or format outside the supported set       */
  MOE_ERR_WORKSPACE = -3,     /* workspace smaller than moe_workspace_bytes()    */
  MOE_ERR_CUDA = -4,          /* a CUDA runtime call failed (see moe_status_str) */
  MOE_ERR_DEVICE_CHECK = -5,  /* a kernel's own check failed (moe_device_status) */
  MOE_ERR_TIMEOUT = -6        /* a bounded device wait gave up                   */
} moe_status;

typedef struct moe_config {
  int32_t num_experts;   /* E                                    */
  int32_t hidden;        /* H                                    */
  int32_t inter;         /* I, intermediate size of each expert  */
  int32_t top_k;         /* k                                    */
  int32_t shared_inter;  /* 0 = no shared expert, else == inter  */
  int32_t bits;          /* 4 or 2                               */
  int32_t block;         /* 32 (4-bit) or 16 (2-bit)             */
  int32_t half_levels;   /* 0: q = c - 2^(bits-1) (integer levels,
                            2-bit ternary); 1: q = c - (2^bits-1)/2,
                            the 2^bits half-integer levels (2-bit:
                            four levels +-1/2, +-3/2)              */
  int32_t scale_fmt;     /* 0: one fp16 scale per block; 1: one E4M3
                            (fp8: sign, 4 exponent bits with bias 7,
                            3 mantissa bits, no infinities, largest
                            finite 448) byte per block, times one
                            fp32 scale per weight row (the
                            *_row_scales arrays); block 32 (4-bit) or
                            16 (2-bit), integer levels only.  Layers with fp8 scales
                            run on the single-launch decode kernel
                            (hidden 2048, inter 768) and on the
                            stand-alone GEMV kernels at every batch
                            size; the tensor-core prefill does not
                            read them.                              */
} moe_config;

/* One layer's weights; every pointer is device memory owned by the caller. */
typedef struct moe_layer_weights {
  const uint8_t*  gate_up_codes;          /* [E][2I][H*bits/8]                  */
  const uint16_t* gate_up_scales;         /* [E][2I][H/block] fp16 bits         */
  const uint8_t*  down_codes;             /* [E][H][I*bits/8]                   */
  const uint16_t* down_scales;            /* [E][H][I/block]                    */
  const uint8_t*  shared_gate_up_codes;   /* [2I][H*bits/8]; NULL if no shared  */
  const uint16_t* shared_gate_up_scales;  /* [2I][H/block]                      */
  const uint8_t*  shared_down_codes;      /* [H][I*bits/8]                      */
  const uint16_t* shared_down_scales;     /* [H][I/block]                       */
  const uint16_t* router_w;               /* [E][H] bf16 bits                   */
  const float*    router_bias;            /* [E] fp32, or NULL (no bias)        */
  const uint16_t* shared_gate_w;          /* [H] bf16 bits: the shared expert's
                                             output is scaled by sigmoid(x . w)
                                             (fp32); NULL = weight 1.  Needs a
                                             shared expert.  Layers with a gate
                                             run on the separate kernels, not
                                             the single-launch decode kernel.  */
  /* scale_fmt = 1 only (NULL otherwise): the *_scales arrays above then hold
   * one E4M3 byte per block (same shapes, one byte per element instead of
   * two), and the weight of element j of row r is q * e4m3(scale byte) *
   * row_scale[r].  fp32, 16-byte aligned (the decode kernels copy them in
   * bulk with the codes). */
  const float*    gate_up_row_scales;     /* [E][2I]                            */
  const float*    down_row_scales;        /* [E][H]                             */
  const float*    shared_gate_up_row_scales;  /* [2I]; NULL if no shared        */
  const float*    shared_down_row_scales;     /* [H]                            */
} moe_layer_weights;

/* Bytes of device workspace needed by moe_route / moe_layer_forward /
 * moe_stack_forward for up to max_tokens tokens.  Returns 0 for an invalid or
 * unsupported config or max_tokens < 0. */
size_t moe_workspace_bytes(const moe_config* cfg, int32_t max_tokens);

/* Router and grouping only (the selection and gate weights of the operation
 * above, plus the per-expert token lists).  Inputs: router_w [E][H] bf16,
 * router_bias [E] or NULL, x [T][H] bf16.  Outputs (device, caller-owned):
 *   topk_idx [T][k] int32 (slots by descending logit), topk_w [T][k] fp32,
 *   expert_counts [E], expert_offsets [E+1] (exclusive prefix sum),
 *   pairs [T*k]: pair ids t*k+j sorted by expert, then by token.
 * Any output pointer may be NULL except topk_idx and topk_w. */
int moe_route(const moe_config* cfg, const uint16_t* router_w, const float* router_bias,
              const uint16_t* x, int32_t T, int32_t* topk_idx, float* topk_w,
              int32_t* expert_counts, int32_t* expert_offsets, int32_t* pairs,
              void* workspace, size_t ws_bytes, void* stream);

/* One MoE layer: y[T][H] (bf16) = out as defined above for x[T][H] (bf16).
 * x and y may not overlap.  T <= 64 takes the decode path (grouped GEMV on
 * CUDA cores); larger T takes the prefill path (grouped tcgen05 GEMMs).  At
 * 32 <= T <= 64 the decode kernel, once it has routed the batch, hands the
 * layer to the prefill kernels when its cost model predicts them faster for
 * that routing (see moe_debug_decode_path); the result is within the same
 * tolerance either way, and the same inputs still give the same output. */
int moe_layer_forward(const moe_config* cfg, const moe_layer_weights* w,
                      const uint16_t* x, int32_t T, uint16_t* y,
                      void* workspace, size_t ws_bytes, void* stream);

/* Expert-parallel share of one MoE layer (one rank of ep_size, experts
 * sharded by e % ep_size == ep_rank).  The pages run every expert of a layer
 * on one machine; splitting the routed experts over GPUs is the one exchange
 * step the layer admits: each rank routes all T tokens (the router is
 * replicated), computes only the pairs whose expert it owns, and the layer
 * output is the sum of the ranks' partials (an all-reduce), rounded to bf16.
 *   y_partial[t][h] (fp32, device, [T][H], owned by the caller) =
 *       [ep_rank == 0] * FFN_shared(x_t)[h]
 *     + sum over j with idx[t][j] % ep_size == ep_rank of w[t][j] * FFN_idx[t][j](x_t)[h]
 * with idx, w and FFN as in moe_layer_forward.  w holds the full expert
 * arrays; only the owned experts' rows (and the shared expert's on rank 0,
 * which other ranks may pass as NULL) are read.  1 <= ep_size <= num_experts,
 * 0 <= ep_rank < ep_size, else MOE_ERR_INVALID_ARG; x and y_partial may not
 * overlap.  Runs the separate route / grouped GEMV or GEMM / combine kernels
 * (not the single-launch decode kernel).  ep_size = 1 gives the whole layer
 * output before its bf16 rounding. */
int moe_layer_forward_ep(const moe_config* cfg, const moe_layer_weights* w,
                         const uint16_t* x, int32_t T, int32_t ep_rank, int32_t ep_size,
                         float* y_partial, void* workspace, size_t ws_bytes, void* stream);

/* L layers in sequence on the residual stream, in place:
 *   for l in 0..L-1:  x <- bf16(x + moe_l(bf16(rmsnorm(x))))
 * rmsnorm(x) = x / sqrt(mean(x^2) + 1e-6) per token (weight 1).
 * layers: HOST array of L weight structs (device pointers inside).
 * topk_trace: NULL, or device int32 [L][T][k] that receives each layer's
 * selection (for validation). */
int moe_stack_forward(const moe_config* cfg, const moe_layer_weights* layers, int32_t L,
                      uint16_t* x_inout, int32_t T, int32_t* topk_trace,
                      void* workspace, size_t ws_bytes, void* stream);

/* Allocation-free variant of moe_layer_forward.  The pages have no
 * counterpart: it exists for callers that cannot allocate device memory
 * themselves -- for example a plugin running inside a host application that
 * has already claimed the GPU's memory through its own pool, or code that must
 * not call cudaMalloc/cudaFree because those calls can synchronise the whole
 * device.  Inputs, outputs and results are those of moe_layer_forward (the
 * same kernels on the same inputs give the same bits), and the arguments are
 * checked in the same order with the same codes; the scratch is a fixed array
 * of MOE_NOALLOC_SCRATCH_BYTES (4 MiB) compiled into libmoe.so, which every
 * GPU that loads the library keeps until the process exits.  If
 * moe_workspace_bytes(cfg, T) exceeds that size the call returns
 * MOE_ERR_WORKSPACE and launches nothing (at the 512-expert, H=2048, I=768,
 * k=10 shape this allows up to 23 tokens).  The first call on a device (and
 * the first after its context was destroyed and re-created, e.g. by
 * cudaDeviceReset) looks up the array's device address with that device
 * current; make that first call before any stream capture.  All calls share
 * the one array and it keeps the previous call's contents (the call clears
 * the part that must start at zero): calls that overlap on the GPU (from other
 * streams or host threads) race, so the caller must serialise them.  No
 * allocating routine is called. */
#define MOE_NOALLOC_SCRATCH_BYTES (4u << 20)
int moe_layer_forward_noalloc(const moe_config* cfg, const moe_layer_weights* w,
                              const uint16_t* x, int32_t T, uint16_t* y, void* stream);

/* The device check word of moe_layer_forward_noalloc's scratch on the current
 * device, as moe_device_status reads it from a workspace (synchronises the
 * device): *code_out = 0 when no kernel of the last call reported a failed
 * check, else the moe_status code (e.g. MOE_ERR_TIMEOUT), and the return value
 * is MOE_ERR_DEVICE_CHECK.  The pages have no counterpart. */
int moe_noalloc_device_status(int32_t* code_out);

/* Reads back the device check word kept in the workspace (synchronises the
 * device).  *code_out = 0 when no kernel reported a failed check. */
int moe_device_status(const void* workspace, int32_t* code_out);

/* Test hook: rows [row0, row0+rows) of a packed matrix with `cols` columns,
 * decoded by the same device routine the GEMV kernels use, written as fp32
 * out[rows][cols].  Not on the timed path.  scale_fmt 0 only; fp8 scales go
 * through moe_dequant_rows_scaled. */
int moe_dequant_rows(const moe_config* cfg, const uint8_t* codes, const uint16_t* scales,
                     int32_t row0, int32_t rows, int32_t cols, float* out, void* stream);

/* The same for either scale format: with cfg->scale_fmt = 1, `scales` holds
 * one E4M3 byte per block and row_scales (device, fp32, indexed by the row of
 * the matrix) is required; with 0 it must be NULL. */
int moe_dequant_rows_scaled(const moe_config* cfg, const uint8_t* codes, const void* scales,
                            const float* row_scales, int32_t row0, int32_t rows, int32_t cols, float* out,
                            void* stream);

/* Measurement hook.  moe_profile_begin(n) makes the next n layer calls
 * record CUDA events around their four phases on the call's stream (route,
 * gate/up + SwiGLU, down, combine); moe_profile_end() waits for those events
 * and returns the summed milliseconds per phase in ms_out[0..3] -- and in
 * ms_out[4] the time of calls that ran as one fused decode kernel -- and the
 * number of recorded calls in *calls.  Events are host-side driver objects; no device
 * memory is allocated.  Not thread-safe; meant for benchmarks. */
int moe_profile_begin(int32_t max_calls);
int moe_profile_end(float* ms_out, int32_t* calls);

/* Measurement hook: while device_buf is non-null, fused decode launches write
 * timestamps of each CTA's first layer to device_buf[cta][32] (zero it first;
 * the caller owns the buffer; null switches it off).  SM clock64 cycles:
 *   [8] layer start, [21] scratch counters cleared, [19] token 0's row loaded,
 *   [20] token 0 staged, [14] token 0's router logits done (with its router
 *   logits when each warp stages one token), [15] this CTA's router logits
 *   written, [0] router logits done (CTA barrier), [1] after the first grid
 *   barrier, [9] top-k done, [10] routing lists done, [2] work lists ready,
 *   [3] gate/up done, [4] after the waits for other CTAs' gate/up rows,
 *   [5] down done, [6] after the second grid barrier, [7] combine done;
 *   consumer group 0: [24] / [25] first gate/up stage's data in / last
 *   gate/up stage done, [26] / [27] the same for down; producer: [28] / [29]
 *   first / last gate/up stage issued, [30] / [31] down.  %globaltimer ns
 *   (comparable across CTAs): [22] layer start, [23] combine done.
 *   [11..13] gate/up and [16..18] down, consumer group 0: ns spent waiting
 *   for stage data, ns spent staging tokens, stages taken.
 * Calls made while it is set are not reentrant-safe measurements of a
 * production run; they only observe one. */
void moe_debug_fused_timing(unsigned long long* device_buf);

/* Measurement hook: while device_buf is non-null, the prefill grouped GEMMs
 * write per-CTA totals to device_buf[pass][cta][16] (pass 0 gate/up, 1 down;
 * cta < the SM count; zero it first; the caller owns it).  Waits are in SM
 * clock cycles:
 *   [0] packed-weight producer waiting for a free stage, [1] token producer
 *   waiting for a free stage, [2] MMA waiting for the A and B operands,
 *   [4] MMA waiting for a free accumulator, [5] dequantizer (first thread)
 *   waiting for packed weights, [6] dequantizer waiting for a free A stage,
 *   [7] epilogue (first thread) waiting for an accumulator, [12] cycles in the
 *   MMA issue blocks, [13] cycles in tile lookups, [15] cycles of the whole
 *   MMA loop; %globaltimer (ns): [8] start and [9] end of the MMA thread, [11]
 *   end of the epilogue; counts: [10] tiles, [14] k-blocks. */
void moe_debug_prefill_timing(unsigned long long* device_buf);

/* Measurement and test hook for single-layer batches of 32..64 tokens, where
 * the single-launch decode kernel routes the batch and then either finishes
 * the layer on the CUDA cores or leaves it to the grouped tensor-core kernels
 * queued behind it, whichever its cost model predicts to be faster (skewed
 * routing puts tens of tokens on a few experts, where the tensor cores win).
 * mode 0: that choice (default); 1: always the CUDA-core kernel; 2: always
 * the tensor-core kernels.  Other values mean 0.  Process-wide, not
 * thread-safe. */
void moe_debug_decode_path(int32_t mode);

/* Failure-path test hook: launches one bounded wait, through the library's
 * own mbarrier wait, on a barrier that never completes.  After the wait's
 * cycle limit (about 1.5 s) the probe records MOE_ERR_TIMEOUT in the status
 * word of `workspace` (device, 256-byte aligned, its first 8 bytes zeroed by
 * the caller; read back with moe_device_status) and returns; the context
 * stays usable.  Asynchronous on `stream`; MOE_ERR_INVALID_ARG for a null or
 * misaligned workspace. */
int moe_debug_wait_probe(void* workspace, void* stream);

/* The cudaError_t value behind the calling thread's most recent
 * MOE_ERR_CUDA (0 if none). */
int moe_last_cuda_error(void);

/* Static description of a status code. */
const char* moe_status_str(int status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_CAPI_H */
