/*
 * gla_oracle.c -- fp64 oracle for the GTR token mixer forward pass.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only tests/, __graft_entry__.smoke()
 * and bench.py's cpu_baseline / reference leg load this library.  It shares no
 * code, header, table or helper with the CUDA path under
 * recurrent_vision_backbone_b200/.
 *
 * What it computes (plain reading of the pages, token by token, no chunking):
 *
 *   GTR news article (tokendh.com), section "线性注意力到底在省什么":
 *   the token mixer is a gated linear attention with a learnable forget gate
 *   that decays the recurrent state on the key side only; the value-side decay
 *   is fixed to 1.  Written out, for one (batch, head) sequence:
 *
 *       a_t = exp(g_t)                       (per key channel, g_t <= 0)
 *       S_t = diag(a_t) S_{t-1} + k_t^T v_t  (S is dk x dv, S_{-1} = S0 or 0)
 *       o_t = q_t S_t                        (inclusive: token t sees its own k v)
 *
 *   Same article, section "单向扫描的致命缺陷，以及GTR怎么补": each block scans
 *   the patch grid in one of four directions (left->right, right->left,
 *   top->bottom, bottom->top).  Reading taken for the mirrored directions:
 *   R->L is L->R on the horizontally mirrored grid (rows top to bottom, each
 *   row right to left); B->T is T->B on the vertically mirrored grid (columns
 *   left to right, each column bottom to top).  T->B is column-major.
 *
 * Layouts (all C-contiguous, fp64):
 *   q, k, g : [B, N, heads, dk]    v, out : [B, N, heads, dv]
 *   s0, s_final : [B, heads, dk, dv]      N = H*W, token n = y*W + x.
 *
 * Parity status: the forward is pinned by tests/test_oracle_pins.py (brute-force closed form,
 * a==1 and a==0 closed forms, direction identities, chunk-size invariance of an
 * independent chunkwise restatement, state passing, linearity, exact rational
 * arithmetic on a hand-sized case); the backward (gla_oracle_bwd, at the end) by
 * tests/test_oracle_bwd.py (central finite differences of the pinned forward, float64
 * autograd of an independent recurrence, the decay-gradient identity, closed forms).
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { DIR_L2R = 0, DIR_R2L = 1, DIR_T2B = 2, DIR_B2T = 3 };

/* Scan position p (0 .. H*W-1) -> memory token index n = y*W + x. */
static long scan_to_token(long p, long H, long W, int direction)
{
    long y, x;
    switch (direction) {
    case DIR_L2R: y = p / W; x = p % W; break;
    case DIR_R2L: y = p / W; x = W - 1 - p % W; break;
    case DIR_T2B: x = p / H; y = p % H; break;
    default:      x = p / H; y = H - 1 - p % H; break; /* DIR_B2T */
    }
    return y * W + x;
}

/*
 * Runs scan positions [p_begin, p_end) of every (b, h) sequence.
 * The state entering position p_begin is s0 (or zero when s0 == NULL);
 * the state after position p_end-1 is written to s_final (when non-NULL).
 * Output rows of tokens outside the range are left untouched.
 * Returns 0 on success, -1 on a bad argument, -2 on allocation failure.
 */
int gla_oracle_fwd_range(const double *q, const double *k, const double *v,
                         const double *g, int B, int heads, int H, int W,
                         int dk, int dv, int direction, long p_begin, long p_end,
                         const double *s0, double *out, double *s_final)
{
    if (!q || !k || !v || !g || !out) return -1;
    if (B < 0 || heads < 0 || H < 0 || W < 0 || dk <= 0 || dv <= 0) return -1;
    if (direction < 0 || direction > 3) return -1;
    const long N = (long)H * (long)W;
    if (p_begin < 0 || p_end < p_begin || p_end > N) return -1;
    const long nseq = (long)B * heads;
    int failed = 0;

#pragma omp parallel for schedule(dynamic, 1)
    for (long sq = 0; sq < nseq; ++sq) {
        const long b = sq / heads, h = sq % heads;
        double *S = (double *)malloc(sizeof(double) * (size_t)dk * (size_t)dv);
        double *a = (double *)malloc(sizeof(double) * (size_t)dk);
        if (!S || !a) {
            free(S);
            free(a);
#pragma omp atomic write
            failed = 1;
            continue;
        }
        if (s0)
            memcpy(S, s0 + sq * (long)dk * dv, sizeof(double) * (size_t)dk * dv);
        else
            memset(S, 0, sizeof(double) * (size_t)dk * dv);

        for (long p = p_begin; p < p_end; ++p) {
            const long n = scan_to_token(p, H, W, direction);
            const long row = (b * N + n) * heads + h;
            const double *qt = q + row * dk, *kt = k + row * dk, *gt = g + row * dk;
            const double *vt = v + row * dv;
            double *ot = out + row * dv;
            for (int i = 0; i < dk; ++i) a[i] = exp(gt[i]);
            /* S <- diag(a) S + k^T v : decay multiplies key rows only. */
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j)
                    S[(long)i * dv + j] = a[i] * S[(long)i * dv + j] + kt[i] * vt[j];
            /* o = q S, read after this token's update. */
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += qt[i] * S[(long)i * dv + j];
                ot[j] = acc;
            }
        }
        if (s_final)
            memcpy(s_final + sq * (long)dk * dv, S, sizeof(double) * (size_t)dk * dv);
        free(S);
        free(a);
    }
    return failed ? -2 : 0;
}

/* Whole scan: positions [0, H*W). */
int gla_oracle_fwd(const double *q, const double *k, const double *v, const double *g,
                   int B, int heads, int H, int W, int dk, int dv, int direction,
                   const double *s0, double *out, double *s_final)
{
    return gla_oracle_fwd_range(q, k, v, g, B, heads, H, W, dk, dv, direction, 0,
                                (long)H * (long)W, s0, out, s_final);
}

/* Scan position -> token index, exported so tests can check the map itself. */
long gla_oracle_scan_to_token(long p, int H, int W, int direction)
{
    if (direction < 0 || direction > 3 || H <= 0 || W <= 0 || p < 0 || p >= (long)H * W)
        return -1;
    return scan_to_token(p, H, W, direction);
}

int gla_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void gla_oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/*
 * Key-side forget gate from its pre-activation z (GTR news article, section
 * "线性注意力到底在省什么": a learnable forget gate on the key side; the gate value is
 * a = sigmoid(z)^(1/tau), so its log-decay is g = log(sigmoid(z)) / tau).
 *
 *   log(sigmoid(z)) = -log(1 + exp(-z))
 *
 * evaluated as min(z, 0) - log1p(exp(-|z|)): the two forms are equal for either sign
 * of z (for z < 0, -log(1 + e^-z) = z - log(e^z + 1)), and this one never overflows.
 * Writes n values of g.  Returns 0, or -1 on a bad argument.
 */
int gla_oracle_gate(const double *z, long n, double tau, double *g)
{
    if ((!z || !g) && n > 0) return -1;
    if (n < 0 || !(tau > 0.0)) return -1;
    for (long i = 0; i < n; ++i) {
        const double x = z[i];
        const double ls = (x < 0.0 ? x : 0.0) - log1p(exp(-fabs(x)));
        g[i] = ls / tau;
    }
    return 0;
}

/*
 * Backward pass of the token mixer (the gradients a training step needs: the GTR news
 * article, section "老师教学生，但只教最后一道题的答案", trains the backbone by
 * distillation with a squared L2 loss on the last layer's patch features; the pages print
 * no backward, so this is plain reverse-mode differentiation of the recurrence above).
 *
 * Given the upstream gradients dO_t = dL/do_t ([B, N, heads, dv]) and dS_f = dL/dS_{N-1}
 * (the final state's gradient, [B, heads, dk, dv], or NULL for zero), with
 * G_t = dL/dS_t the total gradient of the state after position t:
 *
 *       G_{N-1} = dS_f + q_{N-1}^T dO_{N-1}
 *       G_t     = q_t^T dO_t + diag(a_{t+1}) G_{t+1}
 *       dq_t    = S_t dO_t^T                  (dq_t[i] = sum_j S_t[i,j] dO_t[j])
 *       dk_t    = G_t v_t^T                   (dk_t[i] = sum_j G_t[i,j] v_t[j])
 *       dv_t    = k_t G_t                     (dv_t[j] = sum_i k_t[i] G_t[i,j])
 *       dg_t    = a_t * (sum_j G_t[i,j] S_{t-1}[i,j])   (chain rule through a = exp g)
 *       dS0     = diag(a_0) G_0
 *
 * The states S_t are recomputed from fp64 checkpoints taken every kSeg positions on a
 * first forward sweep (the same recurrence, so they are the same numbers), which keeps
 * memory at (N / kSeg + kSeg) states per sequence.  Position order and directions as
 * in gla_oracle_fwd_range.  Outputs: dq, dk, dg [B, N, heads, dk]; dv [B, N, heads, dv];
 * ds0 [B, heads, dk, dv] or NULL.  Returns 0, -1 on a bad argument, -2 on allocation
 * failure.
 */
enum { kSeg = 64 };

int gla_oracle_bwd(const double *q, const double *k, const double *v, const double *g,
                   const double *dout, const double *dsf, int B, int heads, int H, int W,
                   int dk, int dv, int direction, const double *s0, double *dq,
                   double *dk_out, double *dv_out, double *dg, double *ds0)
{
    if (!q || !k || !v || !g || !dout || !dq || !dk_out || !dv_out || !dg) return -1;
    if (B < 0 || heads < 0 || H < 0 || W < 0 || dk <= 0 || dv <= 0) return -1;
    if (direction < 0 || direction > 3) return -1;
    const long N = (long)H * (long)W;
    const long nseq = (long)B * heads;
    const long SZ = (long)dk * dv;
    const long nck = (N + kSeg - 1) / kSeg;
    int failed = 0;

#pragma omp parallel for schedule(dynamic, 1)
    for (long sq = 0; sq < nseq; ++sq) {
        const long b = sq / heads, h = sq % heads;
        double *ck = (double *)malloc(sizeof(double) * (size_t)(nck + 1) * SZ);
        double *seg = (double *)malloc(sizeof(double) * (size_t)(kSeg + 1) * SZ);
        double *G = (double *)malloc(sizeof(double) * (size_t)SZ);
        double *a = (double *)malloc(sizeof(double) * (size_t)dk);
        if (!ck || !seg || !G || !a) {
            free(ck); free(seg); free(G); free(a);
#pragma omp atomic write
            failed = 1;
            continue;
        }
        /* forward sweep: the state entering every segment */
        double *S = seg;
        if (s0) memcpy(S, s0 + sq * SZ, sizeof(double) * (size_t)SZ);
        else memset(S, 0, sizeof(double) * (size_t)SZ);
        for (long p = 0; p < N; ++p) {
            if (p % kSeg == 0) memcpy(ck + (p / kSeg) * SZ, S, sizeof(double) * (size_t)SZ);
            const long row = (b * N + scan_to_token(p, H, W, direction)) * heads + h;
            const double *kt = k + row * dk, *gt = g + row * dk, *vt = v + row * dv;
            for (int i = 0; i < dk; ++i) {
                const double ai = exp(gt[i]);
                for (int j = 0; j < dv; ++j) S[(long)i * dv + j] = ai * S[(long)i * dv + j] + kt[i] * vt[j];
            }
        }
        /* G starts as the final state's gradient */
        if (dsf) memcpy(G, dsf + sq * SZ, sizeof(double) * (size_t)SZ);
        else memset(G, 0, sizeof(double) * (size_t)SZ);
        /* reverse sweep, one segment at a time: recompute its states, then walk back */
        for (long m = nck - 1; m >= 0; --m) {
            const long p0 = m * kSeg, p1 = (p0 + kSeg < N) ? p0 + kSeg : N;
            memcpy(seg, ck + m * SZ, sizeof(double) * (size_t)SZ);   /* seg[0] = S_{p0-1} */
            for (long p = p0; p < p1; ++p) {
                const long row = (b * N + scan_to_token(p, H, W, direction)) * heads + h;
                const double *kt = k + row * dk, *gt = g + row * dk, *vt = v + row * dv;
                const double *Sp = seg + (p - p0) * SZ;
                double *Sn = seg + (p - p0 + 1) * SZ;
                for (int i = 0; i < dk; ++i) {
                    const double ai = exp(gt[i]);
                    for (int j = 0; j < dv; ++j) Sn[(long)i * dv + j] = ai * Sp[(long)i * dv + j] + kt[i] * vt[j];
                }
            }
            for (long p = p1 - 1; p >= p0; --p) {
                const long row = (b * N + scan_to_token(p, H, W, direction)) * heads + h;
                const double *qt = q + row * dk, *kt = k + row * dk, *gt = g + row * dk;
                const double *vt = v + row * dv, *dot = dout + row * dv;
                const double *Sprev = seg + (p - p0) * SZ;    /* S_{p-1} */
                const double *St = seg + (p - p0 + 1) * SZ;   /* S_p */
                /* G_p = (gradient from later positions) + q_p^T dO_p */
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) G[(long)i * dv + j] += qt[i] * dot[j];
                for (int i = 0; i < dk; ++i) {
                    double sq_ = 0.0, sk = 0.0, sa = 0.0;
                    for (int j = 0; j < dv; ++j) {
                        sq_ += St[(long)i * dv + j] * dot[j];
                        sk += G[(long)i * dv + j] * vt[j];
                        sa += G[(long)i * dv + j] * Sprev[(long)i * dv + j];
                    }
                    const double at = exp(gt[i]);   /* a_t of channel i */
                    a[i] = at;
                    dq[row * dk + i] = sq_;
                    dk_out[row * dk + i] = sk;
                    dg[row * dk + i] = at * sa;
                }
                for (int j = 0; j < dv; ++j) {
                    double s = 0.0;
                    for (int i = 0; i < dk; ++i) s += kt[i] * G[(long)i * dv + j];
                    dv_out[row * dv + j] = s;
                }
                /* dL/dS_{p-1} = diag(a_p) G_p */
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) G[(long)i * dv + j] *= a[i];
            }
        }
        if (ds0) memcpy(ds0 + sq * SZ, G, sizeof(double) * (size_t)SZ);
        free(ck); free(seg); free(G); free(a);
    }
    return failed ? -2 : 0;
}
