/*
 * moe_ep.h -- expert-parallel building blocks of libmoe_b200 (C ABI).
 *
 * The pieces a layer whose experts are split over devices needs around its exchange
 * of rows (the pages define a single-device layer; the split rests on its structure:
 * given the routing, each expert's rows are independent): the routed rows of a batch
 * in expert order, the expert FFNs of rows that arrive with their expert, and
 * the combine of expert outputs.  Types, status codes and conventions are those of
 * moe.h; the exchange itself is the caller's (the package's ep module uses NCCL
 * all-to-all through torch.distributed).
 */
#ifndef MOE_EP_H
#define MOE_EP_H

#include "moe.h"

#ifdef __cplusplus
extern "C" {
#endif

/* ---- Expert-parallel building blocks (experts split over devices, each device
 * running the experts it holds on the rows routed to them; the exchange of rows
 * between devices is the caller's, e.g. NCCL all-to-all, as in the
 * package's ep module).  moe_forward of a problem equals, up to the order of its fp32
 * sums, moe_permute of its routing, moe_experts_forward of the permuted rows (each
 * with its expert and weight) and moe_combine of their outputs.  Routed experts only:
 * a shared expert's output enters through moe_combine's shared_output. */

/* The routed rows of a batch in expert order, for routing idx [T, k] (int32) and w
 * [T, k] (fp32) given on the device (moe_route's outputs, or any top-k):
 *   x_perm        [T*k, d] x's dtype: row r is x of the slot it holds (not scaled);
 *                 the rows of expert e are contiguous and token-ascending, experts in
 *                 index order
 *   row_expert    [T*k] int32: row r's expert, modulo experts_per_rank when that is
 *                 positive (its index on the rank holding experts
 *                 [g * experts_per_rank, (g + 1) * experts_per_rank))
 *   row_w         [T*k] fp32: row r's routing weight
 *   expert_counts [E] int32: rows per expert
 *   pos           [T, k] int32: the row of slot (t, j)
 * All device pointers, caller-owned; x and x_perm 16-byte aligned.  experts_per_rank
 * must divide E (0: global indices).  The workspace is moe_workspace_size(shape, opts)
 * bytes, as for moe_forward.  Errors: MOE_ERR_NULL / ARG / ALIGN / WORKSPACE before
 * any launch; an expert index outside [0, E) in idx is MOE_ERR_SHAPE in the workspace
 * status word (moe_debug_status). */
MOE_API int moe_permute(const moe_shape *shape, const moe_options *opts, const int32_t *idx, const float *w,
                        const void *x, void *x_perm, int32_t *row_expert, float *row_w, int32_t *expert_counts,
                        int32_t *pos, int experts_per_rank, void *workspace, size_t workspace_bytes, void *stream);

/* The expert FFNs of rows that arrive with their expert: shape.T rows x [T, d] (in
 * tensors->x), shape.E the experts held here (the stacks in tensors), shape.k = 1,
 * row_expert [T] int32 in [0, E), row_w [T] fp32.  y[r] = row_w[r] * FFN_e(x[r]) as
 * moe_forward's expert outputs (with weigh_inputs: FFN_e(row_w[r] * x[r])), in
 * tensors->y.  Routing options are not used; router_logits, router_weight, topk_idx,
 * topk_w and logits_out must be NULL; no shared expert (Fs = 0).  Otherwise as
 * moe_forward (tensors, workspace, kernel choice, errors). */
MOE_API int moe_experts_forward(const moe_shape *shape, const moe_options *opts, const moe_tensors *tensors,
                                const int32_t *row_expert, const float *row_w, void *workspace,
                                size_t workspace_bytes, void *stream);

/* y[t] = sum_{j<k} Y[pos[t, j]] in fp32 in slot order, + shared_output[t] when given,
 * rounded once to act_dtype ("ClikaRT::nn::QMoEWoQ" forward's combine); Y [rows, d]
 * holds weighted expert outputs (moe_experts_forward's).  Uses shape.T, d, k and
 * act_dtype; pos [T, k] int32 device; Y, y, shared_output 16-byte aligned, y not
 * aliasing an input.  A pos entry outside [0, rows) contributes nothing. */
MOE_API int moe_combine(const moe_shape *shape, const int32_t *pos, const void *Y, int64_t rows,
                        const void *shared_output, void *y, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_EP_H */
