/*
 * gtr_swiglu.h -- C ABI of the gated value branch of GTR's Spatial SwiGLU on B200
 * (sm_100a), in the same library as gtr_gla.h (libgtr_gla.so).
 *
 * GTR news article (tokendh.com), section "单向扫描的致命缺陷，以及GTR怎么补": every
 * GTR block pairs the token mixer with a Spatial SwiGLU, a SwiGLU whose value branch
 * passes through a 3x3 depthwise convolution so that each patch sees its eight grid
 * neighbours directly (a depthwise convolution filters every channel on its own).
 * This call is the fused step between the block's gate/up projections and its down
 * projection (those are plain GEMMs):
 *
 *     out[b,y,x,c] = silu(G[b,y,x,c]) * (bias[c] + sum_{i,j in 0..2} w[c][i][j] * U[b, y+i-1, x+j-1, c])
 *
 * silu(t) = t / (1 + exp(-t)); cross-correlation with zero padding, stride 1 (the
 * output grid is the input grid).  One pass: U and G read once, out written once.
 */
#ifndef GTR_SWIGLU_H
#define GTR_SWIGLU_H

#include "gtr_gla.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Arguments (device pointers, caller-owned; nothing is allocated or freed):
 *   G, U    IEEE binary16 [B, H, W, C], channels contiguous, tokens in grid order
 *           (n = y * W + x): the gate and up projections of the block's input.
 *   w       float32 [C][3][3]: the depthwise kernel, w[c][i][j] weighting the
 *           neighbour at row offset i - 1 and column offset j - 1.
 *   bias    float32 [C] or NULL (no bias).
 *   out     IEEE binary16 [B, H, W, C], round-to-nearest-even of the fp32 result.
 *           It may be G itself (in place); it may not overlap U.
 *   stream  cudaStream_t (NULL: the legacy default stream).  Asynchronous; the call
 *           makes no host wait.
 * Errors: GTR_ERR_INVALID_ARG for negative sizes, NULL required pointers, G, U or
 * out not 16-byte aligned, w or bias not 4-byte aligned, out overlapping U (or G
 * other than exactly), more than 2^34 elements; GTR_ERR_UNSUPPORTED for C not a
 * multiple of 8; GTR_ERR_CUDA for a failed launch.  An empty tensor (any size 0)
 * returns GTR_OK with nothing done.  A result outside the fp16 range sets
 * GTR_ERR_RANGE in the device error word (gtr_gla_device_status).
 */
gtr_status_t gtr_spatial_swiglu_gate(const gtr_half_t *G, const gtr_half_t *U, const float *w,
                                     const float *bias, int B, int H, int W, int C, gtr_half_t *out,
                                     void *stream);

#ifdef __cplusplus
}
#endif

#endif /* GTR_SWIGLU_H */
