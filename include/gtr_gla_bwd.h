/*
 * gtr_gla_bwd.h -- C ABI of the backward pass of the GTR token mixer on B200 (sm_100a).
 *
 * The forward (gtr_gla.h): for one (batch, head) sequence over scan positions t,
 *     S_t = diag(exp g_t) S_{t-1} + k_t^T v_t,   o_t = q_t S_t,   S_{-1} = init_state or 0
 * (GTR news article, tokendh.com, section "线性注意力到底在省什么"; the four scan orders of
 * section "单向扫描的致命缺陷，以及GTR怎么补").  The pages train the backbone by
 * distillation (section "老师教学生，但只教最后一道题的答案") and print no backward: this
 * call returns the gradients of a loss L given its gradients with respect to the
 * forward's outputs,
 *     d_out = dL/do  and  d_final_state = dL/dS_final,
 * namely dL/dq, dL/dk, dL/dv, dL/dg (g the log-decay, as the forward takes it) and
 * dL/d init_state -- exact reverse-mode differentiation of the recurrence, computed
 * chunkwise (64 scan positions per chunk) in FP32 from the FP16 inputs.
 *
 * Layouts (device pointers, C-contiguous, 16-byte aligned), N = Hgrid * Wgrid:
 *     q, k, g            IEEE binary16 [B, N, heads, dk]   (the forward's inputs)
 *     v, d_out           IEEE binary16 [B, N, heads, dv]
 *     init_state         float32 [B, heads, dk, dv] or NULL (zero), as in the forward
 *     d_final_state      float32 [B, heads, dk, dv] or NULL (zero)
 *     grad_q, grad_k, grad_g   float32 [B, N, heads, dk], fully written
 *     grad_v             float32 [B, N, heads, dv], fully written
 *     grad_init_state    float32 [B, heads, dk, dv] or NULL (not wanted)
 * dk is 64 or 128 (128: the recurrence is separable by key channel, so the two halves
 * run one after the other, the second adding its share of grad_v); dv is 64.
 *
 * Ownership and ordering as in gtr_gla.h: every buffer is the caller's, all work is
 * enqueued on `stream`, nothing synchronises the host.  Outputs may not overlap the
 * inputs, each other or the workspace.
 */
#ifndef GTR_GLA_BWD_H
#define GTR_GLA_BWD_H

#include <stddef.h>

#include "gtr_gla.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Bytes of device workspace gtr_gla_bwd needs for a shape: per (sequence, chunk) two
 * 64 x 64 fp32 state tiles (the states entering each chunk and the gradients leaving
 * it) and two 64-float vectors, plus 64 floats per sequence; one key half's worth
 * (halves reuse it).  0 for an empty grid or arguments gtr_gla_bwd would reject.
 * Host-only query.
 */
size_t gtr_gla_bwd_workspace_bytes(int B, int heads, int Hgrid, int Wgrid, int dk, int dv, int chunk);

/*
 * Backward pass of one token-mixer call.
 *   q, k, v, g, init_state, B, heads, Hgrid, Wgrid, dk, dv, direction, chunk:
 *                      as passed to the forward call being differentiated.
 *   d_out, d_final_state, grad_*:  layouts above.
 *   workspace          device memory, 256-byte aligned, at least
 *                      gtr_gla_bwd_workspace_bytes(...) bytes (NULL when that is 0);
 *                      no contents are assumed (every byte read is first written).
 *   workspace_bytes    its size.
 *   stream             cudaStream_t to enqueue on.
 * An empty grid writes grad_init_state = d_final_state (or zeros) and nothing else.
 * Errors: GTR_ERR_INVALID_ARG for null, misaligned, overflowing or overlapping
 * arguments or a short workspace; GTR_ERR_UNSUPPORTED for chunk != 64, dk not in
 * {64, 128} or dv != 64; GTR_ERR_CUDA for a failed launch -- all before or without
 * any partial result being relied on.
 */
gtr_status_t gtr_gla_bwd(const gtr_half_t *q, const gtr_half_t *k, const gtr_half_t *v,
                         const gtr_half_t *g, const gtr_half_t *d_out, const float *init_state,
                         const float *d_final_state, int B, int heads, int Hgrid, int Wgrid,
                         int dk, int dv, int direction, int chunk, float *grad_q, float *grad_k,
                         float *grad_v, float *grad_g, float *grad_init_state, void *workspace,
                         size_t workspace_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* GTR_GLA_BWD_H */
