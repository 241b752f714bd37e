/*
 * jointmoe.h -- C ABI of the MoE feed-forward of a HunyuanImage-3.0 decoder
 * block (forward), for NVIDIA B200 (sm_100a): the fp32 router (softmax over
 * all routed experts, top-k, renormalized), the routed SwiGLU experts as
 * grouped GEMMs over token-sorted rows, the shared SwiGLU expert, and the
 * weighted combine.  Part of libjointattn; the conventions of jointattn.h
 * (status codes, streams, caller-owned buffers, no allocation) hold here.
 *
 * Sources (page title, section / API item):
 *   - HunyuanImage 3.0 Technical Report summary, 3.1.1 Architecture: 64
 *     experts, 8 activated per token, plus one shared MLP.
 *   - hunyuan_image3.model, build_moe_config: softmax over all experts,
 *     top-k, renormalized, one shared expert; HunyuanImage3Block: routed
 *     experts plus the fused shared expert; mlp.gate kept in fp32.
 *   - "HunyuanImage-3.0" model-coverage page, Train: router in fp32
 *     (gate_precision: float32); fused [up; gate] expert projections.
 *   - hunyuan_image3.layers, HunyuanSharedMLP: SwiGLU, gate_and_up_proj holds
 *     [up; gate] with up first, [tokens, hidden] -> [tokens, hidden].
 */
#ifndef JOINTMOE_H
#define JOINTMOE_H

#include <stddef.h>
#include <stdint.h>

#include "jointattn.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Sizes of one MoE feed-forward call. */
typedef struct {
    int32_t T;     /* tokens: rows of x and out, >= 0, < 2^24 */
    int32_t H;     /* hidden size: a multiple of 256 */
    int32_t I;     /* intermediate size of every expert (routed and shared): a multiple of 128 */
    int32_t E;     /* routed experts: 1 <= E <= 80 */
    int32_t topk;  /* experts per token: 1 <= topk <= min(E, 16) */
} hia_moe_dims;

/* Bytes of device workspace hia_moe_fwd needs (256-byte aligned pointer);
 * 0 for invalid dims.  About (T * (topk + 1) + 128 * (E + 1)) rows of
 * (2 H + I) bf16 values plus small tables. */
size_t hia_moe_workspace_bytes(const hia_moe_dims* dims);

/* Forward of the block's MoE feed-forward on `stream`:
 *   logits = x wg^T in fp32 precision (x rounded to bf16 is exact; wg is
 *     split into three bf16 parts whose sum is wg exactly, and the three
 *     products accumulate in fp32 on the tensor cores);
 *   p = softmax(logits) over the E routed experts; the topk largest are
 *     chosen (ties: lower expert index first) and renormalized:
 *     w_j = exp(l_j) / sum over the chosen of exp(l);
 *   out = sum_j w_j * expert_{e_j}(x) + shared(x), with
 *     expert_e(x) = (silu(x W13_e[I:2I]^T) * (x W13_e[0:I]^T)) W2_e^T
 *   computed from bf16 operands with fp32 accumulation; the SwiGLU product
 *   is rounded to bf16 between the two projections and each expert's output
 *   to bf16 before the fp32 weighted sum; out is rounded to bf16.
 * Layouts (row-major, contiguous, device pointers, 16-byte aligned):
 *   x    bf16 [T, H]        the block's normed hidden states
 *   wg   fp32 [E, H]        the router weight
 *   w13  bf16 [E + 1, 2I, H] fused [up; gate] projections, up first; index E
 *                          is the shared expert
 *   w2   bf16 [E + 1, H, I] down projections; index E is the shared expert
 *   out  bf16 [T, H]
 *   topk_ids int32 [T, topk], topk_weights fp32 [T, topk]: the routing
 *     (descending weight); written.
 * Run-to-run the outputs are bitwise identical (each row's result does not
 * depend on where the row sits in the expert-sorted buffers).
 * Errors: HIA_ERR_INVALID_ARG (null pointer with T > 0, dims out of range,
 * short or misaligned workspace), HIA_ERR_UNSUPPORTED (misaligned pointer),
 * HIA_ERR_CUDA, HIA_ERR_DEVICE_TIMEOUT (see hia_get_device_status). */
int hia_moe_fwd(const hia_moe_dims* dims, const void* x, const float* wg, const void* w13, const void* w2,
                void* out, int32_t* topk_ids, float* topk_weights, void* workspace, size_t workspace_bytes,
                void* stream);

#ifdef __cplusplus
}
#endif

#endif /* JOINTMOE_H */
