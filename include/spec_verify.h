/*
 * spec_verify.h -- C ABI of the speculative-verify acceptance step.
 *
 * What it computes. A draft model proposes G tokens per sequence and the
 * main model scores the whole block in one verify pass. Rejection sampling in
 * the verify stage keeps the output distribution of standard decoding
 * (bjdmk.com.cn news on MiMo-V2.5-Pro-UltraSpeed, section
 * "极致协同，通向千速之路", with a block of 8 draft tokens; yifor blog "Xiaomi
 * MiMo and TileRT Push a 1-Trillion-Parameter Model Past 1000 Tokens Per
 * Second on Commodity GPUs", item 2). The rule is the standard
 * speculative-sampling acceptance rule. Per sequence b:
 *
 *   p_i = softmax(target_logits[b][i]),  i = 0 .. G
 *   q_i = softmax(draft_logits[b][i]),   i = 0 .. G-1
 *   for i = 0, 1, ...: accept draft_tokens[b][i] = d when
 *       r_accept[b][i] * q_i(d) < p_i(d)       (d outside [0, V): rejected)
 *   at the first rejection, position n: draw one token from max(0, p_n - q_n)
 *       (from p_n if that is all zero); if all G are accepted, n = G and the
 *       token is drawn from p_G;
 *   a draw from weights w with u = u_sample[b]: the smallest j whose
 *       cumulative weight exceeds u * (total weight).
 *
 * Outputs: n_accepted[b] = n, and tokens_out[b][0 .. G] = d_0 .. d_{n-1}, the
 * drawn token, then -1. The arithmetic is fp64 on the fp32 logits (exp in
 * fp64, sums in fixed orders), so the accept decisions and the draw agree
 * with an fp64 evaluation in any other summation order, except when a value
 * lies within about V * 2^-51 (relative) of its threshold.
 *
 * Layout (all device memory, row-major, no padding):
 *   target_logits fp32 [B][G+1][V]    draft_logits fp32 [B][G][V]
 *   draft_tokens  int32 [B][G]        r_accept fp64 [B][G]    u_sample fp64 [B]
 *   n_accepted    int32 [B]           tokens_out int32 [B][G+1]
 * Logits must be finite or -inf (a masked token). Every row needs at least
 * one finite entry.
 *
 * Ownership and errors. The caller owns every buffer, including the
 * workspace (at least spec_verify_workspace_bytes(B, G, V) bytes of device
 * memory, zero-filled once before its first use and then reused as is).
 * Calls are asynchronous on `stream`, allocate nothing, and may be captured
 * into a CUDA graph. Calls that share one workspace must not run
 * concurrently. Bytes 64..127 of the workspace hold, after a call, eight
 * %globaltimer stamps (ns, uint64), for tracing: the first CTA's start, end
 * of its row statistics, end of the first grid-wide wait, block 0 decided,
 * end of the second wait, end of its weight sums; then the start and the end
 * of the draws (on the last CTA to finish its weight sums).
 * Argument errors (MOE_ERR_INVALID_ARG) are
 * found on the host before any work is enqueued. A device-side wait that ran
 * out is recorded in the workspace and reported by spec_verify_status.
 * Status codes are those of moe_mxfp4.h.
 */
#ifndef SPEC_VERIFY_H
#define SPEC_VERIFY_H

#include "moe_mxfp4.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Upper bounds of the shapes: G draft tokens per block, V vocabulary entries. */
#define SPEC_MAX_GAMMA 16
#define SPEC_MAX_VOCAB (1 << 22)

/*
 * spec_verify_workspace_bytes -- device workspace spec_verify needs for B
 * blocks of G drafts over V tokens (0 < B, 0 <= G <= SPEC_MAX_GAMMA,
 * 0 < V <= SPEC_MAX_VOCAB), or -1 for shapes outside those bounds.
 */
MOE_API int64_t spec_verify_workspace_bytes(int32_t B, int32_t G, int32_t V);

/*
 * spec_verify -- the acceptance step for B verify blocks (layout above), one
 * cooperative launch on `stream`. B == 0 is a no-op. Errors:
 * MOE_ERR_INVALID_ARG (null pointer, shape out of bounds, workspace too
 * small, a pointer not 8-byte aligned), MOE_ERR_DEVICE (no usable device),
 * MOE_ERR_CUDA (the launch failed).
 */
MOE_API int32_t spec_verify(const float* target_logits, const float* draft_logits,
                            const int32_t* draft_tokens, const double* r_accept,
                            const double* u_sample, int32_t B, int32_t G, int32_t V,
                            int32_t* n_accepted, int32_t* tokens_out, void* workspace,
                            int64_t workspace_bytes, void* stream);

/*
 * spec_verify_status -- synchronise `stream`, then return and clear the
 * device-side status kept in the workspace: MOE_OK, or MOE_ERR_TIMEOUT if a
 * grid-wide wait ran out (the outputs of that call are then unspecified;
 * the workspace is usable again). MOE_ERR_CUDA if a CUDA call fails.
 */
MOE_API int32_t spec_verify_status(void* workspace, void* stream);

/*
 * spec_exp -- the fp64 exponential the step evaluates (a table-driven method
 * with about 1 ulp of error), applied to n device values x (x <= 0, the only
 * arguments the step produces) into y, on `stream`; results below -708 are 0.
 * It exists so that its accuracy can be tested against other exp
 * implementations. Errors: MOE_ERR_INVALID_ARG (n < 0, null or misaligned
 * pointers with n > 0), MOE_ERR_DEVICE, MOE_ERR_CUDA.
 */
MOE_API int32_t spec_exp(const double* x, double* y, int64_t n, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SPEC_VERIFY_H */
