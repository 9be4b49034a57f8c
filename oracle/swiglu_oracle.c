/*
 * fp64 oracle of the gated value branch of GTR's Spatial SwiGLU.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE: only tests/, __graft_entry__.smoke() and
 * bench.py's CPU legs load it; it shares no code with the CUDA path.
 *
 * What it follows: GTR news article (tokendh.com), section
 * "单向扫描的致命缺陷，以及GTR怎么补": Spatial SwiGLU is a SwiGLU (a gated linear unit)
 * whose value branch passes through a 3x3 depthwise convolution, so that every patch
 * sees its eight grid neighbours directly; a depthwise convolution filters every
 * channel on its own with its own small kernel.  Plain reading of the parts the page
 * leaves open: the gate is SiLU(x) = x * sigmoid(x) of the gate projection G; the
 * value branch is the up projection U filtered channel by channel with a 3x3 kernel
 * w[c][i][j] (cross-correlation, zero padding, stride 1: the output grid is the
 * input grid) plus an optional per-channel bias; the two are multiplied element by
 * element:
 *
 *     h[b,y,x,c] = silu(G[b,y,x,c]) * (bias[c] + sum_{i,j in 0..2} w[c][i][j] * U[b, y+i-1, x+j-1, c])
 *
 * with U = 0 outside the grid.  G, U, h are [B, H, W, C] (channels contiguous, the
 * tokens in grid order); w is [C][3][3]; bias is [C] or NULL.  Plain loops, in the
 * order of the definition.
 */
#include <math.h>
#include <stddef.h>

static double silu(double x) { return x / (1.0 + exp(-x)); }

int swiglu_oracle_gate_conv(const double *G, const double *U, const double *w, const double *bias,
                            long B, long H, long W, long C, double *h)
{
    if (B < 0 || H < 0 || W < 0 || C < 0) return 1;
    for (long b = 0; b < B; ++b)
        for (long y = 0; y < H; ++y)
            for (long x = 0; x < W; ++x)
                for (long c = 0; c < C; ++c) {
                    double acc = bias ? bias[c] : 0.0;
                    for (long i = 0; i < 3; ++i)
                        for (long j = 0; j < 3; ++j) {
                            const long yy = y + i - 1, xx = x + j - 1;
                            if (yy < 0 || yy >= H || xx < 0 || xx >= W) continue;
                            acc += w[c * 9 + i * 3 + j] * U[((b * H + yy) * W + xx) * C + c];
                        }
                    const long o = ((b * H + y) * W + x) * C + c;
                    h[o] = silu(G[o]) * acc;
                }
    return 0;
}

void swiglu_oracle_silu(const double *x, long n, double *y)
{
    for (long i = 0; i < n; ++i) y[i] = silu(x[i]);
}
