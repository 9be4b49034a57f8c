// gla_bwd.cuh -- backward pass of the GTR token mixer (key-decay gated linear attention)
// for one 64-channel key half and dv = 64 (included by gtr_gla.cu).
//
// The pages train the backbone by distillation (GTR news article, section
// "老师教学生，但只教最后一道题的答案") and print no backward; this is reverse-mode
// differentiation of the recurrence of section "线性注意力到底在省什么",
//     S_t = diag(exp g_t) S_{t-1} + k_t^T v_t,   o_t = q_t S_t,
// given dO = dL/do and dS_f = dL/dS_final, chunkwise with 64 scan positions per chunk.
// Within chunk c (positions t = 0..63, b_t the running sum of g from the chunk start,
// B = b_63, h_c the state entering the chunk, dh_{c+1} = dL/dh_{c+1}):
//
//   K1 (chunk-parallel)  U_c = sum_s (k_s e^{B-b_s})^T v_s,  W_c = sum_t (q_t e^{b_t})^T dO_t
//   K2 (per element, sequential over chunks)
//        h_{c+1} = e^{B_c} h_c + U_c   (h_0 = S0),   dh_c = e^{B_c} dh_{c+1} + W_c (dh_nc = dS_f)
//        dS0 = dh_0;  const = sum_j dS_f[:, j] S_final[:, j]
//   K3 (chunk-parallel), D[t,s] = dO_t . v_s and A[t,s] = sum_i q_t[i] k_s[i] e^{b_t[i]-b_s[i]}
//        for s <= t (zero above the diagonal):
//        dq_t = e^{b_t} (dO_t h_c^T + sum_{s<=t} D[t,s] k_s e^{-b_s})
//        dk_s = e^{B-b_s} (v_s dh_{c+1}^T) + e^{-b_s} sum_{t>=s} D[t,s] q_t e^{b_t}
//        dv_s = sum_{t>=s} A[t,s] dO_t + (k_s e^{B-b_s}) dh_{c+1}
//        x_t = q_t dq_t - k_t dk_t, its suffix sum inside the chunk, and the chunk total
//   K4 (chunk-parallel)  dg_r = sum_{t >= r} x_t + const: the chunk's suffix sums plus the
//        totals of the later chunks.
// dg follows from the loss depending on g only through the running sums b: d/db_t of
// q_t e^{b_t} gives q_t dq_t, of k_t e^{-b_t} gives -k_t dk_t, and the final state adds
// its own term to every position.
//
// Key channels whose chunk decay is below e^-60 ("slow" channels) would overflow the
// factored form e^{b_t} e^{-b_s}; their intra-chunk terms are formed with one exponential
// per (t, s) pair instead.  Arithmetic is fp32 on the CUDA cores (the products are
// register-tiled 64 x 64 x 64 contractions out of shared memory).
#pragma once

namespace gtr {
namespace bw {

constexpr int kC = 64;                 // chunk length
constexpr int kLd = 65;                // shared row stride (floats): conflict-free columns
constexpr int kMat = kC * kLd;         // floats per shared 64 x 64 matrix
constexpr int kThreads = 256;
constexpr float kFastRange = 60.f;     // chunk log-decay above which e^{-b} stays finite

struct Args {
    const __half *q, *k, *g;     // [rows][ldk], at the key half
    const __half *v, *dout;      // [rows][64]
    const float *s0, *dsf;       // [n_seq][sstride] at the key half (row i at i * 64), or null
    float *dq, *dk, *dg;         // [rows][ldk], at the key half
    float *dv;                   // [rows][64]
    float *ds0;                  // like s0, or null
    float *hs, *dhs;             // workspace: [n_seq][nc][64][64] U -> h_c, W -> dh_{c+1}
    float *bc, *xc;              // workspace: [n_seq][nc][64] chunk log-decay, chunk x totals
    float *cst;                  // workspace: [n_seq][64]
    int heads, H, W, N, dir, n_seq, nc, ldk, sstride;
    int acc_dv;                  // 1: add to dv (the second key half)
};

// Token row of scan position p of sequence seq, or -1 past the grid.
__device__ __forceinline__ int bwd_row(const Args &a, int seq, int p) {
    if (p >= a.N) return -1;
    const int bb = seq / a.heads, hh = seq - bb * a.heads;
    return (bb * a.N + scan_to_token(p, a.H, a.W, a.dir)) * a.heads + hh;
}

// 64 rows x 64 fp16 channels (row r at token row rows[r], pitch ld) -> fp32 dst[r][c];
// rows past the grid are zero.
__device__ __forceinline__ void load_tile_h(const __half *src, int ld, const int *rows, float *dst) {
    for (int x = threadIdx.x; x < kC * 8; x += kThreads) {
        const int r = x >> 3, c8 = x & 7, ro = rows[r];
        float f[8];
        if (ro >= 0) {
            const uint4 u = *reinterpret_cast<const uint4 *>(src + (size_t)ro * ld + 8 * c8);
            const __half2 *h2 = reinterpret_cast<const __half2 *>(&u);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 p = __half22float2(h2[e]);
                f[2 * e] = p.x;
                f[2 * e + 1] = p.y;
            }
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = 0.f;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) dst[r * kLd + 8 * c8 + e] = f[e];
    }
}

// A 64 x 64 fp32 matrix, row-major in global memory -> dst[r][c].
__device__ __forceinline__ void load_tile_f(const float *src, float *dst) {
    for (int x = threadIdx.x; x < kC * 16; x += kThreads) {
        const int r = x >> 4, c4 = x & 15;
        const float4 u = *reinterpret_cast<const float4 *>(src + r * 64 + 4 * c4);
        dst[r * kLd + 4 * c4] = u.x;
        dst[r * kLd + 4 * c4 + 1] = u.y;
        dst[r * kLd + 4 * c4 + 2] = u.z;
        dst[r * kLd + 4 * c4 + 3] = u.w;
    }
}

// Running sum of g down each channel (64 threads): b[t][i] over the chunk; returns B.
__device__ __forceinline__ void chunk_cumsum(float *b, float *Bv) {
    if (threadIdx.x < kC) {
        const int i = threadIdx.x;
        float s = 0.f;
        for (int t = 0; t < kC; ++t) {
            s += b[t * kLd + i];
            b[t * kLd + i] = s;
        }
        Bv[i] = s;
    }
}

// Register tile of a 64 x 64 product: thread (ty, tx) = (tid / 16, tid % 16) owns rows
// ty + 16 a and columns tx + 16 b.  Operand element (r, k) of a row-major matrix M is
// M[r * kLd + k]; of a transposed one, M[k * kLd + r].
template <bool kTA, bool kTB>
__device__ __forceinline__ void mm_acc(const float *A, const float *B, float (&acc)[4][4]) {
    const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
#pragma unroll 4
    for (int kk = 0; kk < kC; ++kk) {
        float a[4], b[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int r = ty + 16 * u, c = tx + 16 * u;
            a[u] = kTA ? A[kk * kLd + r] : A[r * kLd + kk];
            b[u] = kTB ? B[c * kLd + kk] : B[kk * kLd + c];
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int w = 0; w < 4; ++w) acc[u][w] = fmaf(a[u], b[w], acc[u][w]);
    }
}

__device__ __forceinline__ void zero4x4(float (&acc)[4][4]) {
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w) acc[u][w] = 0.f;
}

// ---------------------------------------------------------------- K1: chunk locals
// grid n_seq * nc, 256 threads; shared: k, q, b, v, dO (5 matrices) + rows.
__global__ void __launch_bounds__(kThreads) gla_bwd_local_kernel(const Args a) {
    extern __shared__ float smf[];
    float *ks = smf, *qs = ks + kMat, *bs = qs + kMat, *vs = bs + kMat, *ds = vs + kMat;
    __shared__ int rows[kC];
    __shared__ float Bv[kC];
    const int tid = threadIdx.x;
    const int seq = (int)(blockIdx.x / a.nc), c = (int)(blockIdx.x % a.nc);
    if (tid < kC) rows[tid] = bwd_row(a, seq, c * kC + tid);
    __syncthreads();
    load_tile_h(a.k, a.ldk, rows, ks);
    load_tile_h(a.q, a.ldk, rows, qs);
    load_tile_h(a.g, a.ldk, rows, bs);
    load_tile_h(a.v, 64, rows, vs);
    load_tile_h(a.dout, 64, rows, ds);
    __syncthreads();
    chunk_cumsum(bs, Bv);
    __syncthreads();
    const size_t cidx = (size_t)seq * a.nc + c;
    if (tid < kC) a.bc[cidx * kC + tid] = Bv[tid];
    for (int e = tid; e < kC * kC; e += kThreads) {
        const int t = e >> 6, i = e & 63;
        const float b = bs[t * kLd + i];
        ks[t * kLd + i] *= __expf(Bv[i] - b);   // k_s e^{B - b_s} (<= k)
        qs[t * kLd + i] *= __expf(b);           // q_t e^{b_t}     (<= q)
    }
    __syncthreads();
    float u[4][4], w[4][4];
    zero4x4(u);
    zero4x4(w);
    mm_acc<true, false>(ks, vs, u);   // U[i][j] = sum_s kB[s][i] v[s][j]
    mm_acc<true, false>(qs, ds, w);   // W[i][j] = sum_t qe[t][i] dO[t][j]
    const int ty = tid >> 4, tx = tid & 15;
    float *uo = a.hs + cidx * 4096, *wo = a.dhs + cidx * 4096;
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            uo[(ty + 16 * p) * 64 + tx + 16 * r] = u[p][r];
            wo[(ty + 16 * p) * 64 + tx + 16 * r] = w[p][r];
        }
}

// ---------------------------------------------------------------- K2: chunk scans
// grid n_seq * 16, 256 threads: thread e of the sequence's 4096 state elements
// (i = e / 64, j = e % 64).  Loads run kPre chunks ahead of the chain.
constexpr int kPre = 8;

__global__ void __launch_bounds__(kThreads) gla_bwd_scan_kernel(const Args a) {
    __shared__ float red[kThreads / 32];
    const int seq = (int)(blockIdx.x / 16);
    const int e = (int)(blockIdx.x % 16) * kThreads + threadIdx.x, i = e >> 6;
    const int nc = a.nc;
    const size_t base = (size_t)seq * nc * 4096 + e;
    const float *bc = a.bc + (size_t)seq * nc * kC + i;
    const size_t so = (size_t)seq * a.sstride + e;   // (i, j) at i * 64 + j
    // forward: U_c -> h_c (the state entering chunk c)
    float h = a.s0 ? a.s0[so] : 0.f;
    for (int c0 = 0; c0 < nc; c0 += kPre) {
        float uu[kPre], dd[kPre];
#pragma unroll
        for (int r = 0; r < kPre; ++r)
            if (c0 + r < nc) {
                uu[r] = a.hs[base + (size_t)(c0 + r) * 4096];
                dd[r] = __expf(bc[(size_t)(c0 + r) * kC]);
            }
#pragma unroll
        for (int r = 0; r < kPre; ++r)
            if (c0 + r < nc) {
                a.hs[base + (size_t)(c0 + r) * 4096] = h;
                h = fmaf(dd[r], h, uu[r]);
            }
    }
    // const[i] = sum_j dS_f[i][j] S_final[i][j]: the row's 64 elements are warps 2 r, 2 r + 1
    float pr = a.dsf ? a.dsf[so] * h : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) pr += __shfl_xor_sync(0xffffffffu, pr, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = pr;
    __syncthreads();
    if (threadIdx.x < kThreads / 64) {
        const int r = threadIdx.x;
        a.cst[(size_t)seq * kC + (blockIdx.x % 16) * 4 + r] = red[2 * r] + red[2 * r + 1];
    }
    // reverse: W_c -> dh_{c+1} (the gradient of the state leaving chunk c)
    float d = a.dsf ? a.dsf[so] : 0.f;
    for (int c1 = nc - 1; c1 >= 0; c1 -= kPre) {
        float ww[kPre], dd[kPre];
#pragma unroll
        for (int r = 0; r < kPre; ++r)
            if (c1 - r >= 0) {
                ww[r] = a.dhs[base + (size_t)(c1 - r) * 4096];
                dd[r] = __expf(bc[(size_t)(c1 - r) * kC]);
            }
#pragma unroll
        for (int r = 0; r < kPre; ++r)
            if (c1 - r >= 0) {
                a.dhs[base + (size_t)(c1 - r) * 4096] = d;
                d = fmaf(dd[r], d, ww[r]);
            }
    }
    if (a.ds0) a.ds0[so] = d;
}

// ---------------------------------------------------------------- K3: chunk gradients
// grid n_seq * nc, 256 threads; shared: 12 matrices + vectors.
enum { M_Q = 0, M_K, M_B, M_V, M_DO, M_HC, M_DH, M_D, M_A, M_QH, M_KH, M_KB, kGradMats };
constexpr size_t kGradSmem = (size_t)kGradMats * kMat * sizeof(float);

__global__ void __launch_bounds__(kThreads) gla_bwd_grad_kernel(const Args a) {
    extern __shared__ float smf[];
    float *qs = smf + M_Q * kMat, *ks = smf + M_K * kMat, *bs = smf + M_B * kMat;
    float *vs = smf + M_V * kMat, *ds = smf + M_DO * kMat, *hc = smf + M_HC * kMat;
    float *dh = smf + M_DH * kMat, *Dm = smf + M_D * kMat, *Am = smf + M_A * kMat;
    float *qh = smf + M_QH * kMat, *kh = smf + M_KH * kMat, *kB = smf + M_KB * kMat;
    __shared__ int rows[kC];
    __shared__ float Bv[kC];
    __shared__ int fast[kC];
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const int seq = (int)(blockIdx.x / a.nc), c = (int)(blockIdx.x % a.nc);
    const size_t cidx = (size_t)seq * a.nc + c;
    if (tid < kC) rows[tid] = bwd_row(a, seq, c * kC + tid);
    __syncthreads();
    load_tile_h(a.q, a.ldk, rows, qs);
    load_tile_h(a.k, a.ldk, rows, ks);
    load_tile_h(a.g, a.ldk, rows, bs);
    load_tile_h(a.v, 64, rows, vs);
    load_tile_h(a.dout, 64, rows, ds);
    load_tile_f(a.hs + cidx * 4096, hc);
    load_tile_f(a.dhs + cidx * 4096, dh);
    __syncthreads();
    chunk_cumsum(bs, Bv);
    __syncthreads();
    if (tid < kC) fast[tid] = Bv[tid] >= -kFastRange;
    __syncthreads();
    const bool any_slow = __syncthreads_or(tid < kC && !fast[tid]) != 0;
    for (int e = tid; e < kC * kC; e += kThreads) {
        const int t = e >> 6, i = e & 63;
        const float b = bs[t * kLd + i], q = qs[t * kLd + i], k = ks[t * kLd + i];
        const bool f = fast[i] != 0;
        qh[t * kLd + i] = f ? q * __expf(b) : 0.f;
        kh[t * kLd + i] = f ? k * __expf(-b) : 0.f;
        kB[t * kLd + i] = k * __expf(Bv[i] - b);
    }
    __syncthreads();
    // D = dO V^T and A = Qh Kh^T (rows t, columns s), zero above the diagonal
    {
        float d[4][4], m[4][4];
        zero4x4(d);
        zero4x4(m);
        mm_acc<false, true>(ds, vs, d);
        mm_acc<false, true>(qh, kh, m);
#pragma unroll
        for (int p = 0; p < 4; ++p)
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int t = ty + 16 * p, s = tx + 16 * r;
                Dm[t * kLd + s] = s <= t ? d[p][r] : 0.f;
                Am[t * kLd + s] = s <= t ? m[p][r] : 0.f;
            }
    }
    __syncthreads();
    if (any_slow) {   // slow channels' share of A, one exponential per pair
        for (int e = tid; e < kC * kC; e += kThreads) {
            const int t = e >> 6, s = e & 63;
            if (s > t) continue;
            float acc = 0.f;
            for (int i = 0; i < kC; ++i)
                if (!fast[i])
                    acc += qs[t * kLd + i] * ks[s * kLd + i] * __expf(bs[t * kLd + i] - bs[s * kLd + i]);
            Am[t * kLd + s] += acc;
        }
        __syncthreads();
    }
    // dv (rows s, columns j) straight to global memory
    {
        float acc[4][4];
        zero4x4(acc);
        mm_acc<true, false>(Am, ds, acc);   // sum_t A[t][s] dO[t][j]
        mm_acc<false, false>(kB, dh, acc);  // sum_i kB[s][i] dh[i][j]
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const int s = ty + 16 * p, ro = rows[s];
            if (ro < 0) continue;
            float *dst = a.dv + (size_t)ro * 64;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int j = tx + 16 * r;
                dst[j] = a.acc_dv ? dst[j] + acc[p][r] : acc[p][r];
            }
        }
    }
    // dq (rows t, channels i) and dk (rows s, channels i), kept in registers until the
    // shared tiles they replace are free
    float xq[4][4], y1[4][4], y2[4][4];
    zero4x4(xq);
    zero4x4(y1);
    zero4x4(y2);
    mm_acc<false, true>(ds, hc, xq);    // sum_j dO[t][j] h_c[i][j]
    mm_acc<false, false>(Dm, kh, xq);   // sum_s D[t][s] kh[s][i]
    mm_acc<false, true>(vs, dh, y1);    // sum_j v[s][j] dh[i][j]
    mm_acc<true, false>(Dm, qh, y2);    // sum_t D[t][s] qh[t][i]
    __syncthreads();   // every product is done: hc and vs now hold dq and dk
    float *dqs = hc, *dks = vs;
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int t = ty + 16 * p, i = tx + 16 * r;
            const float b = bs[t * kLd + i];
            dqs[t * kLd + i] = __expf(b) * xq[p][r];
            dks[t * kLd + i] = __expf(Bv[i] - b) * y1[p][r] + (fast[i] ? __expf(-b) * y2[p][r] : 0.f);
        }
    __syncthreads();
    if (any_slow) {   // slow channels' intra-chunk terms of dq and dk
        for (int e = tid; e < kC * kC; e += kThreads) {
            const int t = e >> 6, i = e & 63;
            if (fast[i]) continue;
            const float bt = bs[t * kLd + i];
            float sq = 0.f, sk = 0.f;
            for (int s = 0; s <= t; ++s)   // dq: s <= t
                sq += Dm[t * kLd + s] * ks[s * kLd + i] * __expf(bt - bs[s * kLd + i]);
            for (int u = t; u < kC; ++u)   // dk of row t: later rows u >= t
                sk += Dm[u * kLd + t] * qs[u * kLd + i] * __expf(bs[u * kLd + i] - bt);
            dqs[t * kLd + i] += sq;
            dks[t * kLd + i] += sk;
        }
        __syncthreads();
    }
    // x = q dq - k dk, suffix sums down each channel (Am is free)
    float *xs = Am;
    for (int e = tid; e < kC * kC; e += kThreads) {
        const int t = e >> 6, i = e & 63;
        xs[t * kLd + i] = qs[t * kLd + i] * dqs[t * kLd + i] - ks[t * kLd + i] * dks[t * kLd + i];
    }
    __syncthreads();
    if (tid < kC) {
        float s = 0.f;
        for (int t = kC - 1; t >= 0; --t) {
            s += xs[t * kLd + tid];
            xs[t * kLd + tid] = s;
        }
        a.xc[cidx * kC + tid] = s;
    }
    __syncthreads();
    // rows of dq, dk and the chunk part of dg: four threads per row, 16 channels each
    {
        const int t = tid >> 2, c0 = 16 * (tid & 3), ro = rows[t];
        if (ro >= 0) {
            float *oq = a.dq + (size_t)ro * a.ldk, *ok = a.dk + (size_t)ro * a.ldk, *og = a.dg + (size_t)ro * a.ldk;
#pragma unroll
            for (int i4 = 0; i4 < 4; ++i4) {
                const int i = c0 + 4 * i4;
                *reinterpret_cast<float4 *>(oq + i) = make_float4(dqs[t * kLd + i], dqs[t * kLd + i + 1],
                                                                  dqs[t * kLd + i + 2], dqs[t * kLd + i + 3]);
                *reinterpret_cast<float4 *>(ok + i) = make_float4(dks[t * kLd + i], dks[t * kLd + i + 1],
                                                                  dks[t * kLd + i + 2], dks[t * kLd + i + 3]);
                *reinterpret_cast<float4 *>(og + i) = make_float4(xs[t * kLd + i], xs[t * kLd + i + 1],
                                                                  xs[t * kLd + i + 2], xs[t * kLd + i + 3]);
            }
        }
    }
}

// ---------------------------------------------------------------- K4: dg offsets
// grid n_seq * nc, 64 threads (one per channel): dg of the chunk's rows += const + the
// x totals of the later chunks of the sequence.
__global__ void __launch_bounds__(kC) gla_bwd_dg_kernel(const Args a) {
    const int i = threadIdx.x;
    const int seq = (int)(blockIdx.x / a.nc), c = (int)(blockIdx.x % a.nc);
    float off = a.cst[(size_t)seq * kC + i];
    const float *xc = a.xc + (size_t)seq * a.nc * kC + i;
    for (int c2 = c + 1; c2 < a.nc; ++c2) off += xc[(size_t)c2 * kC];
    const int nrows = min(kC, a.N - c * kC);
    for (int t = 0; t < nrows; ++t) {
        const int ro = bwd_row(a, seq, c * kC + t);
        a.dg[(size_t)ro * a.ldk + i] += off;
    }
}

}  // namespace bw
}  // namespace gtr
