/*
 * moe_mxfp4.h -- C ABI of the decode-time MoE expert feed-forward with MXFP4
 * expert weights (B200 / sm_100a).
 *
 * What it computes.  One MoE layer per call of the expert weights stored in
 * MXFP4 (4 bits per expert parameter; the MiMo-V2.5-Pro-UltraSpeed / TileRT
 * pages: bjdmk.com.cn news, section "极致协同，通向千速之路", and the yifor
 * blog digest "Xiaomi MiMo and TileRT Push a 1-Trillion-Parameter Model Past
 * 1000 Tokens Per Second on Commodity GPUs", section "三層協同設計"), applied to
 * the small token block of a speculative-decoding verify step (draft block
 * size 8, so about 9 tokens per sequence: bjdmk.com.cn news, same section).
 * The pages give no formula; the library takes the plain MoE reading:
 *
 *   logits = x Wr^T + b                      (fp64 accumulation, see moe_route)
 *   idx    = the top_k experts by logit, descending, ties to the lower index
 *   w      = softmax(logits)[idx] / sum      (renormalised over the top_k)
 *   y_t    = sum_slot w_slot * Wd_e (silu(Wg_e x_t) * (Wu_e x_t)),  e = idx[t][slot]
 *
 * with Wg, Wu, Wd dequantised exactly from MXFP4 and fp32 accumulation.  With
 * num_layers > 1 the layers run back to back in one launch, each layer's bf16
 * output going through RMSNorm (unit gamma, eps = cfg.rms_eps, no residual)
 * and bf16 rounding to become the next layer's input.  The pages put a
 * persistent engine kernel around this (TileRT blog "Breaking 1000 TPS",
 * section "第一次跃迁：Execution Model Revolution"): moe_forward is one
 * cooperative launch of such a kernel.
 *
 * MXFP4 (OCP Microscaling v1.0): 32-element blocks along the contraction
 * dimension K; each element an E2M1 code (bit 3 sign, bits 2..0 index into
 * {0, 0.5, 1, 1.5, 2, 3, 4, 6}), element 2j in the LOW nibble of byte j; one
 * E8M0 scale byte per block, value 2^(byte-127), byte 255 = NaN.
 *
 * Conventions for every entry point below.
 *  - Pointers named *_host are host memory; every other pointer is DEVICE
 *    memory of the current CUDA device, row-major and contiguous, 16-byte
 *    aligned.  The caller keeps ownership of everything it passes.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Device work
 *    is enqueued asynchronously on it; only moe_status, moe_forward_host and
 *    moe_mxfp4_create (which waits for its repack) synchronise.
 *  - Return value: moe_status_t (0 = MOE_OK).  Argument errors are detected on
 *    the host before any work is enqueued.  Errors detected on the device
 *    (a bounded wait that ran out) are recorded in the handle and reported by
 *    the next moe_status call.  No entry point aborts, throws or prints.
 */
#ifndef MOE_MXFP4_H
#define MOE_MXFP4_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,       /* null pointer, size out of range, misaligned pointer */
  MOE_ERR_UNSUPPORTED_SHAPE = 2, /* a shape the kernels do not tile (see moe_mxfp4_create) */
  MOE_ERR_OOM = 3,               /* device allocation failed in moe_mxfp4_create */
  MOE_ERR_CUDA = 4,              /* a CUDA runtime call or launch failed */
  MOE_ERR_TIMEOUT = 5,           /* a device-side wait exceeded its bound (reported by moe_status) */
  MOE_ERR_DEVICE = 6             /* no usable device, or the engine cannot be co-resident */
} moe_status_t;

typedef struct moe_mxfp4 moe_mxfp4_t; /* opaque handle */

typedef struct {
  int32_t hidden;      /* H: multiple of 128, at most 8192 */
  int32_t inter;       /* I: expert intermediate size, multiple of 128 */
  int32_t num_experts; /* E: 1 .. 512 */
  int32_t top_k;       /* k: 1 .. min(E, 32) */
  int32_t max_tokens;  /* largest T any call will pass, >= 1 */
  int32_t num_layers;  /* 1 .. 16 layers chained inside one moe_forward */
  float rms_eps;       /* RMSNorm epsilon between chained layers (e.g. 1e-6) */
} moe_config_t;

/*
 * mxfp4_quantize -- MXFP4-quantise bf16 weights w_bf16 [rows][K] (K % 32 == 0).
 * Per 32-element block along K: s = max(floor(log2 amax) - 2, -127), scale
 * byte s + 127; each code is the input's sign bit and the nearest E2M1
 * magnitude of |w| / 2^s (ties to the even code, saturating at 6).  A block
 * holding an Inf or NaN gets scale byte 255 and all-zero codes.
 * Output codes [rows][K/2] (element 2j in the low nibble), scales [rows][K/32].
 * rows == 0 is a no-op.  Errors: MOE_ERR_INVALID_ARG for null pointers with
 * rows > 0, rows < 0, K <= 0 or K % 32 != 0; MOE_ERR_CUDA if the launch fails.
 */
MOE_API int32_t mxfp4_quantize(const void* w_bf16, int64_t rows, int64_t K, uint8_t* codes,
                       uint8_t* scales, void* stream);

/*
 * moe_mxfp4_create -- build a handle that owns device copies of num_layers
 * MoE layers, repacked for the weight stream, plus all workspace for calls
 * with up to cfg->max_tokens tokens.
 * Per layer l (host arrays of num_layers DEVICE pointers):
 *   gate_codes[l], up_codes[l]   [E][I][H/2],  gate_scales[l], up_scales[l] [E][I][H/32]
 *   down_codes[l]                [E][H][I/2],  down_scales[l]               [E][H][I/32]
 *   router_w[l]                  [E][H] fp32;  router_bias == NULL or router_bias[l] == NULL
 *                                              means no bias, else [E] fp32.
 * The inputs are read on `stream`; the call synchronises `stream` before it
 * returns, after which the caller may free them.  *out is set to NULL on error.
 * Errors: MOE_ERR_INVALID_ARG (null pointers, cfg fields out of range, device
 * pointers not 16-byte aligned), MOE_ERR_UNSUPPORTED_SHAPE (H or I not a
 * multiple of 128, H > 8192, E > 512, top_k > 32), MOE_ERR_OOM, MOE_ERR_CUDA,
 * MOE_ERR_DEVICE (no device, or the engine kernel does not fit on an SM).
 */
MOE_API int32_t moe_mxfp4_create(const moe_config_t* cfg,
                         const uint8_t* const* gate_codes, const uint8_t* const* gate_scales,
                         const uint8_t* const* up_codes, const uint8_t* const* up_scales,
                         const uint8_t* const* down_codes, const uint8_t* const* down_scales,
                         const float* const* router_w, const float* const* router_bias,
                         void* stream, moe_mxfp4_t** out);

/*
 * moe_route -- routing and permutation of layer `layer` for x_bf16 [T][H]:
 *   topk_idx [T][k] int32   experts in descending-logit order (ties: lower index)
 *   topk_w   [T][k] fp32    softmax over all E, renormalised over the k
 *   counts   [E]    int32   pairs routed to each expert
 *   offsets  [E+1]  int32   exclusive prefix sum of counts
 *   perm     [T*k]  int32   pair id p = t*k + slot at each permuted position;
 *                           each expert's segment is in ascending p
 *   inv_perm [T*k]  int32   position of each pair id
 * Logits are accumulated in fp64 from exact bf16 x fp32 products, so the
 * selection agrees with an exact computation except on logit gaps below about
 * 1e-10.  T == 0 is a no-op.  Errors: MOE_ERR_INVALID_ARG (null handle or
 * pointers, layer out of range, T < 0 or T > max_tokens), MOE_ERR_CUDA.
 */
MOE_API int32_t moe_route(moe_mxfp4_t* h, int32_t layer, const void* x_bf16, int32_t T,
                  int32_t* topk_idx, float* topk_w, int32_t* counts, int32_t* offsets,
                  int32_t* perm, int32_t* inv_perm, void* stream);

/*
 * moe_forward -- y_bf16 [T][H] = the chain of num_layers MoE layers on
 * x_bf16 [T][H], in ONE cooperative launch on `stream`.  layer_io_bf16 is
 * NULL or a [num_layers+1][T][H] bf16 buffer that receives every layer's
 * input (slot l) and the final output (slot num_layers).  x and y may not
 * overlap.  T == 0 is a no-op.  Errors: MOE_ERR_INVALID_ARG, MOE_ERR_CUDA;
 * device-side timeouts are reported by the next moe_status.  The call only
 * enqueues the launch (no synchronisation, no host reads of device memory),
 * so it may be captured into a CUDA graph; calls on one handle must not run
 * concurrently (they share its workspace).
 */
MOE_API int32_t moe_forward(moe_mxfp4_t* h, const void* x_bf16, int32_t T, void* y_bf16,
                    void* layer_io_bf16, void* stream);

/*
 * moe_forward_partial -- one layer (a handle of num_layers == 1) with the
 * output left as the fp32 sum over the k slots, in slot order, without the
 * bf16 rounding: y_f32 [T][H] (device, 16-byte aligned).  It is one rank's
 * share of an I-sharded layer. A handle built on rows [r*I/N, (r+1)*I/N) of
 * every expert's gate and up matrices, and on the same columns of its down
 * matrix (with their block scales), routes exactly as the unsharded layer.
 * SwiGLU acts per intermediate row, so the N ranks' partials sum to the
 * layer's output. moe_round_bf16 of that sum gives moe_forward's result, up to
 * the fp32 summation order. With N = 1 it gives that result bit for bit. The
 * sum over ranks is an all-reduce; the pages' deployment is one 8-GPU node
 * (HyperAI salon transcript "Speed is Intelligence", GLM-5.1 case; bjdmk
 * news, 8 GPUs per node). Arguments and capture safety as for moe_forward.
 * The handle's bf16 staging output serves as scratch, and it is also slot 0
 * of moe_forward_host_async. So order the call after any such copies still in
 * flight (moe_host_join on `stream`). Errors: MOE_ERR_INVALID_ARG,
 * MOE_ERR_UNSUPPORTED_SHAPE (num_layers != 1), MOE_ERR_CUDA.
 */
MOE_API int32_t moe_forward_partial(moe_mxfp4_t* h, const void* x_bf16, int32_t T, float* y_f32,
                                    void* stream);

/*
 * The I-sharded layer with a fused one-shot all-reduce.  The pages' deployment
 * is one node of 8 GPUs (HyperAI salon transcript "Speed is Intelligence",
 * GLM-5.1 case; bjdmk.com.cn news, section "1T模型，千token每秒"); splitting
 * every expert's intermediate dimension over the GPUs gives each the same
 * share of every hit expert's bytes whatever the routing skew, and leaves one
 * exchange: the sum of the per-rank partial outputs.  Instead of a separate
 * all-reduce launch, the engine's last combine does it: each rank writes its
 * fp32 partial into its own region, publishes the call's epoch into every
 * rank's region (system-scope release), waits until its own region holds the
 * epoch from every rank (bounded; a timeout is MOE_ERR_TIMEOUT at moe_status),
 * and sums the ranks' partials in rank order with plain loads of the peers'
 * memory (NVLink), then rounds to bf16.  Every rank's y is bit-identical.
 * No multicast copy is involved.
 *
 * Set-up, once per handle (a handle of num_layers == 1 built on the rank's
 * I-slice, see moe_forward_partial):
 *   moe_ishard_region      the handle's region: MAX_RANKS epoch words, then two
 *                          slots of [max_tokens][hidden] fp32 (allocated and
 *                          zeroed on the first call; synchronises the device).
 *   moe_ishard_ipc_handle  its 64-byte CUDA IPC handle, to send to the peers.
 *   moe_ishard_ipc_open    map a peer's region (from its handle) on the current
 *                          device; moe_ishard_ipc_close unmaps it.
 *   moe_ishard_attach      rank, world (1..8) and every rank's region as the
 *                          current device addresses it (regions[rank] must be
 *                          this handle's own); restarts the epochs and clears
 *                          this region's epoch words (synchronises the device),
 *                          so every rank must attach before any rank calls
 *                          (a barrier over the ranks), also after a timeout.
 * Then moe_forward_ishard(h, x, T, y) on every rank, the same calls in the same
 * order (each call is one epoch).  x must be the same on every rank.  Errors:
 * MOE_ERR_INVALID_ARG (null or misaligned pointers, rank/world out of range,
 * not attached), MOE_ERR_UNSUPPORTED_SHAPE (num_layers != 1), MOE_ERR_OOM,
 * MOE_ERR_CUDA.
 */
#define MOE_IPC_HANDLE_BYTES 64
MOE_API int32_t moe_ishard_region(moe_mxfp4_t* h, void** base_out, uint64_t* bytes_out);
MOE_API int32_t moe_ishard_ipc_handle(moe_mxfp4_t* h, void* handle_out);
MOE_API int32_t moe_ishard_ipc_open(const void* handle, void** base_out);
MOE_API int32_t moe_ishard_ipc_close(void* base);
MOE_API int32_t moe_ishard_attach(moe_mxfp4_t* h, int32_t rank, int32_t world, void* const* regions);
MOE_API int32_t moe_forward_ishard(moe_mxfp4_t* h, const void* x_bf16, int32_t T, void* y_bf16,
                                   void* stream);

/*
 * moe_round_bf16 -- out_bf16[i] = bf16(in_f32[i]) (round to nearest even) for
 * n device values on `stream`; the last step of an I-sharded layer, after the
 * partial outputs were summed.  Errors: MOE_ERR_INVALID_ARG (n < 0; null or
 * misaligned pointers with n > 0), MOE_ERR_CUDA.
 */
MOE_API int32_t moe_round_bf16(const float* in_f32, void* out_bf16, int64_t n, void* stream);

/*
 * moe_forward_host -- moe_forward with HOST input and output: copies
 * x_host [T][H] bf16 to the handle's device staging buffer, runs the layers,
 * copies y back to y_host [T][H] and synchronises `stream`.  Pinned host
 * memory gives asynchronous copies; pageable memory works too.  Its staging
 * buffers are slot 0 of moe_forward_host_async, whose copies and layers in
 * flight it waits for first.  Returns the first error, device-side errors
 * included.
 */
MOE_API int32_t moe_forward_host(moe_mxfp4_t* h, const void* x_host, int32_t T, void* y_host,
                         void* stream);

/*
 * moe_forward_host_async -- moe_forward with HOST input and output, without
 * synchronising: the copy of x_host to one of two device staging slots (on
 * an internal copy stream), the layers (on `stream`) and the copy of y back
 * to y_host (on a second internal copy stream) are only enqueued, so a call's
 * copies overlap the layers of its neighbours.  x_host must stay unchanged
 * and y_host unread until the copies are done: moe_host_join, then a
 * synchronisation of `stream` (or moe_status, which synchronises the copy
 * streams too).  Pinned host memory gives the overlap; pageable memory works
 * but serialises.  Errors: MOE_ERR_INVALID_ARG, MOE_ERR_CUDA; device-side
 * timeouts are reported by the next moe_status.
 */
MOE_API int32_t moe_forward_host_async(moe_mxfp4_t* h, const void* x_host, int32_t T, void* y_host,
                               void* stream);

/*
 * moe_host_join -- make `stream` wait (without blocking the host) for the
 * output copies of every moe_forward_host_async call enqueued so far.
 */
MOE_API int32_t moe_host_join(moe_mxfp4_t* h, void* stream);

/*
 * moe_forward_ops -- the layers of moe_forward, operator by operator: per
 * layer six launches on `stream` (router partial logits; routing by one CTA;
 * x term images; gate/up + SwiGLU jobs; down jobs; combine, + RMSNorm between
 * layers), each one CTA per SM except the routing (one CTA) and an RMSNorm
 * combine (one CTA per token).  The results are bit-identical to moe_forward.
 * It is the baseline the single persistent launch is measured against: the
 * execution-model passages (TileRT blog "Breaking 1000 TPS", section on the
 * execution model; HyperAI salon transcript "Speed is Intelligence", section
 * on CUDA Graph and PDL) set a resident engine against operator-by-operator
 * launches with CUDA graphs and programmatic dependent launch.
 * flags: MOE_OPS_PDL launches every kernel as a programmatic dependent of its
 * predecessor (it is scheduled while the predecessor drains, then waits for
 * it before touching any data).  Arguments, layout and capture safety as for
 * moe_forward.  Only T*K <= 256 (the verify-block sizes);
 * larger calls return MOE_ERR_UNSUPPORTED_SHAPE.  Errors: MOE_ERR_INVALID_ARG,
 * MOE_ERR_UNSUPPORTED_SHAPE, MOE_ERR_CUDA; device-side timeouts are reported
 * by the next moe_status.
 */
#define MOE_OPS_PDL 1
MOE_API int32_t moe_forward_ops(moe_mxfp4_t* h, const void* x_bf16, int32_t T, void* y_bf16,
                                void* layer_io_bf16, int32_t flags, void* stream);

/*
 * moe_status -- synchronise `stream`, then return and clear the device-side
 * status of the handle: MOE_OK, or MOE_ERR_TIMEOUT if a bounded wait inside
 * the engine expired (the handle's wait state is reset, so it stays usable).
 * MOE_ERR_CUDA if the synchronisation itself fails.
 */
MOE_API int32_t moe_status(moe_mxfp4_t* h, void* stream);

/*
 * moe_phase_ns -- tracing: synchronise `stream`, then write to the HOST array
 * ns_out up to max_n durations (ns, %globaltimer of CTA 0) of the last
 * moe_forward of the handle, seven per layer, as seen by CTA 0: router
 * logits; x term images (T*K <= 256: after arriving at the routing barrier);
 * the wait for the routing; top-k (T*K <= 256: the copy of the routing
 * tables); permutation + unit tables (+ tile gather); the MXFP4 weight
 * stream; combine (+ RMSNorm).
 * Values of a launch that stopped early are unspecified.
 */
MOE_API int32_t moe_phase_ns(moe_mxfp4_t* h, uint64_t* ns_out, int32_t max_n, void* stream);

/*
 * moe_stream_profile -- tracing of the weight stream: synchronise `stream`,
 * copy up to max_n counters accumulated since the previous call to the HOST
 * array out (may be NULL when max_n == 0), reset them, and switch counting on
 * (enable != 0) or off for the following launches.  Counters, in SM clock
 * cycles summed over CTAs (and over the 8 epilogue warps for the epilogue
 * ones): producer waiting for free ring slots, producer waiting for gate/up
 * completion, producer total, stages issued; MMA issuer waiting for stage
 * data, issuing (scale copies + MMAs), waiting for a free accumulator;
 * epilogue waiting for accumulators, epilogue work, epilogue total; jobs.
 */
MOE_API int32_t moe_stream_profile(moe_mxfp4_t* h, int32_t enable, uint64_t* out, int32_t max_n,
                                   void* stream);

/*
 * moe_set_large_kind -- the weight stream used when a call has many positions
 * per expert (T*K > 256 and T*K >= 8*E): 1 = E2M1 term tiles on the block-
 * scaled fp4 tensor-core MMA (x and the SwiGLU output expanded into five
 * E2M1 terms; with at most 24 positions per expert and hidden % 256 == 0,
 * jobs of two row blocks share each activation stage), 2 = bf16 tiles on the
 * bf16 tensor-core MMA (MXFP4 weights dequantised to bf16 in shared memory, x
 * exact, the SwiGLU output as two bf16 terms), 3 = E4M3 term tiles on the
 * block-scaled kind that takes E2M1 weights and E4M3 activations (the MXFP4
 * weight codes rewritten in shared memory into that kind's 16-byte-chunk
 * form; x as two E4M3 terms, the SwiGLU output as three).  Default 1.  The
 * kinds are the ablation of the MXFP4 tensor-core paths (bjdmk.com.cn news,
 * section "极致协同，通向千速之路", on MXFP4 for the experts; TileRT blog
 * "Breaking 1000 TPS", section "第一次跃迁：Execution Model Revolution", on
 * the tensor cores under the tile pipeline).  Errors: MOE_ERR_INVALID_ARG.
 */
MOE_API int32_t moe_set_large_kind(moe_mxfp4_t* h, int32_t kind);

/* moe_set_timeout_ns -- bound of every device-side wait (default 2 s; env MOE_TIMEOUT_NS). */
MOE_API int32_t moe_set_timeout_ns(moe_mxfp4_t* h, uint64_t ns);

/* moe_engine_grid -- CTAs of one engine launch (one per SM on B200), or 0 for a NULL handle. */
MOE_API int32_t moe_engine_grid(const moe_mxfp4_t* h);

/* moe_mxfp4_destroy -- free every device allocation of the handle (NULL is a no-op).
 * Work already enqueued on the handle must have finished. */
MOE_API void moe_mxfp4_destroy(moe_mxfp4_t* h);

/*
 * moe_route_static -- moe_route without a handle and without any device
 * allocation.  No counterpart on the pages: it exists for callers that cannot
 * call cudaMalloc (a caching allocator that already owns the free memory, a
 * process whose memory budget was reserved up front, a serving path where
 * allocation is forbidden) but need the router.  Same outputs and output
 * layouts as moe_route, for router_w [num_experts][hidden] fp32 and
 * router_bias [num_experts] fp32 or NULL, both DEVICE pointers.
 * Working memory: one static device array of MOE_ROUTE_STATIC_SCRATCH_BYTES
 * that every device using the library holds until the process exits.  The
 * first call on a device resolves that array's device address (and sets the
 * kernel's shared-memory limit); make that first call before any stream
 * capture.  All calls share the array: calls whose kernels overlap on the GPU
 * race and give wrong outputs, so serialise them.  The call clears the words
 * that must start at zero itself.  The working memory of a call is
 * 64*T*num_experts + 36*min(num_experts, T*top_k) + 17*T*top_k bytes plus
 * under 2 KB of alignment (fp64 partial logits, unit tables, barrier words):
 * T up to about 1000 at num_experts = 128, top_k = 8.  Larger sizes return
 * MOE_ERR_UNSUPPORTED_SHAPE; hidden must be a multiple of 128 (at most 8192),
 * num_experts <= 512, top_k <= min(num_experts, 32).  T == 0 is a no-op.
 * A device-side wait that runs out (bound: 2 s, or env MOE_TIMEOUT_NS) leaves
 * the outputs undefined; moe_route_static_status reports it.
 */
#define MOE_ROUTE_STATIC_SCRATCH_BYTES (8u << 20)
MOE_API int32_t moe_route_static(const void* x_bf16, int32_t T, int32_t hidden,
                                 const float* router_w, const float* router_bias,
                                 int32_t num_experts, int32_t top_k, int32_t* topk_idx,
                                 float* topk_w, int32_t* counts, int32_t* offsets, int32_t* perm,
                                 int32_t* inv_perm, void* stream);

/*
 * moe_route_static_status -- synchronise `stream`, then return and clear the
 * device-side status of the moe_route_static calls made on the current device:
 * MOE_OK, or MOE_ERR_TIMEOUT if a bounded wait of the last such call ran out
 * (its outputs are then undefined).  It allocates nothing either.  MOE_OK when
 * no call was made on this device; MOE_ERR_CUDA if the synchronisation or the
 * read of the status word fails.
 */
MOE_API int32_t moe_route_static_status(void* stream);

/* moe_status_str -- static English text for a status code. */
MOE_API const char* moe_status_str(int32_t status);

#ifdef __cplusplus
}
#endif
#endif /* MOE_MXFP4_H */
