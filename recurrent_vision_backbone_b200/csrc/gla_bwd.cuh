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
constexpr int kLd = 68;                // shared row stride (floats): 16-byte rows for vector loads
constexpr int kMat = kC * kLd;         // floats per shared 64 x 64 matrix
constexpr int kThreads = 256;
constexpr float kFastRange = 60.f;     // chunk log-decay above which e^{-b} stays finite
// A log-decay at or below this is a gate of 0 (exp(g) < 2e-35).  Inside a chunk the
// running sum of g is kept as (number of such gates so far, sum of the other g's), so
// that a gate of 0 (g = -inf) costs no precision in the decays after it: the decay
// between positions s <= t is exp(R_t - R_s) if no zero gate lies between them, else 0.
constexpr float kZeroGate = -80.f;

struct Args {
    const __half *q, *k, *g;     // [rows][ldk], at the key half
    const __half *v, *dout;      // [rows][64]
    const float *s0, *dsf;       // [n_seq][sstride] at the key half (row i at i * 64), or null
    float *dq, *dk, *dg;         // [rows][ldk], at the key half
    float *dv;                   // [rows][64]
    float *ds0;                  // like s0, or null
    float *hs, *dhs;             // workspace: U -> h_c, W -> dh_{c+1} tiles (layout: tile_idx)
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

// Workspace position of element e = i * 64 + j of sequence seq's chunk-c state tile:
// [seq][e / 32][chunk][e % 32], so that one warp's 32 elements over consecutive chunks
// are consecutive 128-byte lines (the scans walk the chunks; the chunk kernels still
// read or write whole 128-byte lines).
__device__ __forceinline__ size_t tile_idx(int nc, int seq, int c, int e) {
    return (((size_t)seq * 128 + (e >> 5)) * nc + c) * 32 + (e & 31);
}

// Keeps the compiler from moving memory accesses across this point: the loads issued
// before it are all in flight before the first one is waited for.
__device__ __forceinline__ void issue_fence() { asm volatile("" ::: "memory"); }

// 64 rows x 64 fp16 channels (row r at token row rows[r], pitch ld): this thread's two
// 16-byte pieces (x = tid, tid + 256: row x / 8, channels 8 (x % 8) ..), zero past the
// grid; then stored as fp32 into dst[r][c].
struct HalfTile {
    uint4 p[2];
};
__device__ __forceinline__ void issue_tile_h(const __half *src, int ld, const int *rows, HalfTile &t) {
#pragma unroll
    for (int m = 0; m < 2; ++m) {
        const int x = threadIdx.x + kThreads * m, ro = rows[x >> 3];
        t.p[m] = ro >= 0 ? *reinterpret_cast<const uint4 *>(src + (size_t)ro * ld + 8 * (x & 7))
                         : make_uint4(0u, 0u, 0u, 0u);
    }
}
__device__ __forceinline__ void store_tile_h(const HalfTile &t, float *dst) {
#pragma unroll
    for (int m = 0; m < 2; ++m) {
        const int x = threadIdx.x + kThreads * m;
        const __half2 *h2 = reinterpret_cast<const __half2 *>(&t.p[m]);
        const float2 f0 = __half22float2(h2[0]), f1 = __half22float2(h2[1]);
        const float2 f2 = __half22float2(h2[2]), f3 = __half22float2(h2[3]);
        float4 *d4 = reinterpret_cast<float4 *>(dst + (x >> 3) * kLd + 8 * (x & 7));
        d4[0] = make_float4(f0.x, f0.y, f1.x, f1.y);
        d4[1] = make_float4(f2.x, f2.y, f3.x, f3.y);
    }
}

// A chunk's 64 x 64 fp32 state tile from the workspace: this thread's four 16-byte
// pieces (elements 4 x .. 4 x + 3, x = tid + 256 m), then stored into dst[i][j].
struct StateTile {
    float4 p[4];
};
__device__ __forceinline__ void issue_state_tile(const float *src, int nc, int seq, int c, StateTile &t) {
#pragma unroll
    for (int m = 0; m < 4; ++m)
        t.p[m] = *reinterpret_cast<const float4 *>(src + tile_idx(nc, seq, c, 4 * (threadIdx.x + kThreads * m)));
}
__device__ __forceinline__ void store_state_tile(const StateTile &t, float *dst) {
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int e = 4 * (threadIdx.x + kThreads * m);
        *reinterpret_cast<float4 *>(dst + (e >> 6) * kLd + (e & 63)) = t.p[m];
    }
}

// Running sums of g down each channel (64 threads), as the count of zero gates kz[t][i]
// and the sum R[t][i] of the other g's over rows 0..t (R written over g in b); Kv, Bv:
// the chunk's totals.  The column is read into registers first, so the chain is
// register adds only.
__device__ __forceinline__ void chunk_cumsum(float *b, float *kz, float *Bv, float *Kv) {
    if (threadIdx.x < kC) {
        const int i = threadIdx.x;
        float col[kC];
#pragma unroll
        for (int t = 0; t < kC; ++t) col[t] = b[t * kLd + i];
        float s = 0.f, n = 0.f;
#pragma unroll
        for (int t = 0; t < kC; ++t) {
            if (col[t] <= kZeroGate) n += 1.f;
            else s += col[t];
            b[t * kLd + i] = s;
            kz[t * kLd + i] = n;
        }
        Bv[i] = s;
        Kv[i] = n;
    }
}

// e^{b_t - b_s} for rows s <= t of channel i (0 across a zero gate)
__device__ __forceinline__ float decay_ts(const float *R, const float *kz, int t, int s, int i) {
    return kz[t * kLd + i] == kz[s * kLd + i] ? __expf(fminf(R[t * kLd + i] - R[s * kLd + i], 0.f)) : 0.f;
}
// e^{B - b_s}: from row s to the chunk's end
__device__ __forceinline__ float decay_to_end(const float *R, const float *kz, const float *Bv, const float *Kv,
                                              int s, int i) {
    return Kv[i] == kz[s * kLd + i] ? __expf(Bv[i] - R[s * kLd + i]) : 0.f;
}
// e^{b_t}: from the chunk's start to row t
__device__ __forceinline__ float decay_from_start(const float *R, const float *kz, int t, int i) {
    return kz[t * kLd + i] == 0.f ? __expf(R[t * kLd + i]) : 0.f;
}

// Register tile of a 64 x 64 product, k in steps of four: thread (ty, tx) = (tid / 16,
// tid % 16) owns rows 4 ty + u and columns 4 tx + w (kColVec) or tx + 16 w.  Operand
// element (r, k) of a row-major matrix M is M[r * kLd + k]; of a transposed one,
// M[k * kLd + r].  Every A read is a 16-byte vector (four k of one row, or four rows of
// one k); B reads are vectors where its layout and the column mapping line up (rows of
// a transposed B with columns tx + 16 w; a row-major B with columns 4 tx + w).
__device__ __forceinline__ int mm_row(int u) { return 4 * (threadIdx.x >> 4) + u; }
template <bool kColVec>
__device__ __forceinline__ int mm_col(int w) {
    const int tx = threadIdx.x & 15;
    return kColVec ? 4 * tx + w : tx + 16 * w;
}

template <bool kTA, bool kTB, bool kColVec>
__device__ __forceinline__ void mm_acc(const float *A, const float *B, float (&acc)[4][4]) {
    const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
#pragma unroll 2
    for (int kk = 0; kk < kC; kk += 4) {
        float a[4][4], b[4][4];   // a[u][q]: row u, k = kk + q;  b[q][w]: k = kk + q, column w
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            if (kTA) {
                const float4 v = *reinterpret_cast<const float4 *>(A + (kk + x) * kLd + 4 * ty);
                a[0][x] = v.x; a[1][x] = v.y; a[2][x] = v.z; a[3][x] = v.w;
            } else {
                const float4 v = *reinterpret_cast<const float4 *>(A + (4 * ty + x) * kLd + kk);
                a[x][0] = v.x; a[x][1] = v.y; a[x][2] = v.z; a[x][3] = v.w;
            }
        }
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            if (kTB && !kColVec) {
                const float4 v = *reinterpret_cast<const float4 *>(B + (tx + 16 * x) * kLd + kk);
                b[0][x] = v.x; b[1][x] = v.y; b[2][x] = v.z; b[3][x] = v.w;
            } else if (!kTB && kColVec) {
                const float4 v = *reinterpret_cast<const float4 *>(B + (kk + x) * kLd + 4 * tx);
                b[x][0] = v.x; b[x][1] = v.y; b[x][2] = v.z; b[x][3] = v.w;
            } else {
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const int c = mm_col<kColVec>(w);
                    b[x][w] = kTB ? B[c * kLd + kk + x] : B[(kk + x) * kLd + c];
                }
            }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int w = 0; w < 4; ++w) acc[u][w] = fmaf(a[u][q], b[q][w], acc[u][w]);
    }
}

__device__ __forceinline__ void zero4x4(float (&acc)[4][4]) {
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w) acc[u][w] = 0.f;
}

// ---------------------------------------------------------------- K1: chunk locals
// grid n_seq * nc, 256 threads; shared: k, q, b, v, dO, zero-gate counts (6 matrices).
constexpr size_t kLocalSmem = 6 * (size_t)kMat * sizeof(float);
__global__ void __launch_bounds__(kThreads) gla_bwd_local_kernel(const Args a) {
    extern __shared__ float smf[];
    float *ks = smf, *qs = ks + kMat, *bs = qs + kMat, *vs = bs + kMat, *ds = vs + kMat, *kz = ds + kMat;
    __shared__ int rows[kC];
    __shared__ float Bv[kC], Kv[kC];
    const int tid = threadIdx.x;
    const int seq = (int)(blockIdx.x / a.nc), c = (int)(blockIdx.x % a.nc);
    if (tid < kC) rows[tid] = bwd_row(a, seq, c * kC + tid);
    __syncthreads();
    {
        HalfTile tk, tq, tg, tv, td;   // every load in flight before the first store
        issue_tile_h(a.k, a.ldk, rows, tk);
        issue_tile_h(a.q, a.ldk, rows, tq);
        issue_tile_h(a.g, a.ldk, rows, tg);
        issue_tile_h(a.v, 64, rows, tv);
        issue_tile_h(a.dout, 64, rows, td);
        issue_fence();
        store_tile_h(tk, ks);
        store_tile_h(tq, qs);
        store_tile_h(tg, bs);
        store_tile_h(tv, vs);
        store_tile_h(td, ds);
    }
    __syncthreads();
    chunk_cumsum(bs, kz, Bv, Kv);
    __syncthreads();
    const size_t cidx = (size_t)seq * a.nc + c;
    if (tid < kC) a.bc[cidx * kC + tid] = Kv[tid] == 0.f ? Bv[tid] : -1e30f;   // log of e^B (0 past a zero gate)
    for (int e = tid; e < kC * kC; e += kThreads) {
        const int t = e >> 6, i = e & 63;
        ks[t * kLd + i] *= decay_to_end(bs, kz, Bv, Kv, t, i);   // k_s e^{B - b_s} (<= k)
        qs[t * kLd + i] *= decay_from_start(bs, kz, t, i);        // q_t e^{b_t}     (<= q)
    }
    __syncthreads();
    float u[4][4], w[4][4];
    zero4x4(u);
    zero4x4(w);
    mm_acc<true, false, true>(ks, vs, u);   // U[i][j] = sum_s kB[s][i] v[s][j]
    mm_acc<true, false, true>(qs, ds, w);   // W[i][j] = sum_t qe[t][i] dO[t][j]
#pragma unroll
    for (int p = 0; p < 4; ++p) {   // columns 4 tx .. 4 tx + 3: one 16-byte store each
        const size_t o = tile_idx(a.nc, seq, c, mm_row(p) * 64 + mm_col<true>(0));
        *reinterpret_cast<float4 *>(a.hs + o) = make_float4(u[p][0], u[p][1], u[p][2], u[p][3]);
        *reinterpret_cast<float4 *>(a.dhs + o) = make_float4(w[p][0], w[p][1], w[p][2], w[p][3]);
    }
}

// ---------------------------------------------------------------- K2: chunk scans
// grid n_seq * 16, 256 threads: thread e of the sequence's 4096 state elements
// (i = e / 64, j = e % 64), walking the chunks in batches of kPre: every load of a
// batch is in flight before the chain uses the first (one memory latency per batch).
constexpr int kPre = 32;

__global__ void __launch_bounds__(kThreads) gla_bwd_scan_kernel(const Args a) {
    __shared__ float red[kThreads / 32];
    const int seq = (int)(blockIdx.x / 16);
    const int e = (int)(blockIdx.x % 16) * kThreads + threadIdx.x, i = e >> 6;
    const int nc = a.nc;
    const size_t base = tile_idx(nc, seq, 0, e);   // + 32 per chunk
    const float *bc = a.bc + (size_t)seq * nc * kC + i;
    const size_t so = (size_t)seq * a.sstride + e;   // (i, j) at i * 64 + j
    // forward: U_c -> h_c (the state entering chunk c)
    float h = a.s0 ? a.s0[so] : 0.f;
    for (int c0 = 0; c0 < nc; c0 += kPre) {
        float uu[kPre], dd[kPre];
#pragma unroll
        for (int r = 0; r < kPre; ++r)
            if (c0 + r < nc) {
                uu[r] = a.hs[base + (size_t)(c0 + r) * 32];
                dd[r] = bc[(size_t)(c0 + r) * kC];
            }
        issue_fence();
#pragma unroll
        for (int r = 0; r < kPre; ++r)
            if (c0 + r < nc) {
                a.hs[base + (size_t)(c0 + r) * 32] = h;
                h = fmaf(__expf(dd[r]), h, uu[r]);
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
                ww[r] = a.dhs[base + (size_t)(c1 - r) * 32];
                dd[r] = bc[(size_t)(c1 - r) * kC];
            }
        issue_fence();
#pragma unroll
        for (int r = 0; r < kPre; ++r)
            if (c1 - r >= 0) {
                a.dhs[base + (size_t)(c1 - r) * 32] = d;
                d = fmaf(__expf(dd[r]), d, ww[r]);
            }
    }
    if (a.ds0) a.ds0[so] = d;
}

// ---------------------------------------------------------------- K3: chunk gradients
// grid n_seq * nc, 256 threads; shared: 12 matrices + vectors.
enum { M_Q = 0, M_K, M_B, M_V, M_DO, M_HC, M_DH, M_D, M_A, M_QH, M_KH, M_KB, M_KZ, kGradMats };
constexpr size_t kGradSmem = (size_t)kGradMats * kMat * sizeof(float);

__global__ void __launch_bounds__(kThreads, 1) gla_bwd_grad_kernel(const Args a) {   // one CTA per SM (shared memory)
    extern __shared__ float smf[];
    float *qs = smf + M_Q * kMat, *ks = smf + M_K * kMat, *bs = smf + M_B * kMat;
    float *vs = smf + M_V * kMat, *ds = smf + M_DO * kMat, *hc = smf + M_HC * kMat;
    float *dh = smf + M_DH * kMat, *Dm = smf + M_D * kMat, *Am = smf + M_A * kMat;
    float *qh = smf + M_QH * kMat, *kh = smf + M_KH * kMat, *kB = smf + M_KB * kMat;
    float *kz = smf + M_KZ * kMat;
    __shared__ int rows[kC];
    __shared__ float Bv[kC], Kv[kC];
    __shared__ int fast[kC];
    const int tid = threadIdx.x;
    const int seq = (int)(blockIdx.x / a.nc), c = (int)(blockIdx.x % a.nc);
    const size_t cidx = (size_t)seq * a.nc + c;
    if (tid < kC) rows[tid] = bwd_row(a, seq, c * kC + tid);
    __syncthreads();
    {
        HalfTile tq, tk, tg, tv, td;   // every load in flight before the first store
        StateTile th, tdh;
        issue_tile_h(a.q, a.ldk, rows, tq);
        issue_tile_h(a.k, a.ldk, rows, tk);
        issue_tile_h(a.g, a.ldk, rows, tg);
        issue_tile_h(a.v, 64, rows, tv);
        issue_tile_h(a.dout, 64, rows, td);
        issue_state_tile(a.hs, a.nc, seq, c, th);
        issue_state_tile(a.dhs, a.nc, seq, c, tdh);
        issue_fence();
        store_tile_h(tq, qs);
        store_tile_h(tk, ks);
        store_tile_h(tg, bs);
        store_tile_h(tv, vs);
        store_tile_h(td, ds);
        store_state_tile(th, hc);
        store_state_tile(tdh, dh);
    }
    __syncthreads();
    chunk_cumsum(bs, kz, Bv, Kv);
    __syncthreads();
    if (tid < kC) fast[tid] = Kv[tid] == 0.f && Bv[tid] >= -kFastRange;
    __syncthreads();
    const bool any_slow = __syncthreads_or(tid < kC && !fast[tid]) != 0;
    for (int e = tid; e < kC * kC; e += kThreads) {
        const int t = e >> 6, i = e & 63;
        const float b = bs[t * kLd + i], q = qs[t * kLd + i], k = ks[t * kLd + i];
        const bool f = fast[i] != 0;   // (no zero gate in the chunk: b = R)
        qh[t * kLd + i] = f ? q * __expf(b) : 0.f;
        kh[t * kLd + i] = f ? k * __expf(-b) : 0.f;
        kB[t * kLd + i] = k * decay_to_end(bs, kz, Bv, Kv, t, i);
    }
    __syncthreads();
    // D = dO V^T and A = Qh Kh^T (rows t, columns s), zero above the diagonal
    {
        float d[4][4], m[4][4];
        zero4x4(d);
        zero4x4(m);
        mm_acc<false, true, false>(ds, vs, d);
        mm_acc<false, true, false>(qh, kh, m);
#pragma unroll
        for (int p = 0; p < 4; ++p)
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int t = mm_row(p), s = mm_col<false>(r);
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
                if (!fast[i]) acc += qs[t * kLd + i] * ks[s * kLd + i] * decay_ts(bs, kz, t, s, i);
            Am[t * kLd + s] += acc;
        }
        __syncthreads();
    }
    // dv (rows s, columns j) straight to global memory
    {
        float acc[4][4];
        zero4x4(acc);
        mm_acc<true, false, true>(Am, ds, acc);    // sum_t A[t][s] dO[t][j]
        mm_acc<false, false, true>(kB, dh, acc);   // sum_i kB[s][i] dh[i][j]
#pragma unroll
        for (int p = 0; p < 4; ++p) {   // columns 4 tx .. 4 tx + 3 of row s: one 16-byte access
            const int s = mm_row(p), ro = rows[s];
            if (ro < 0) continue;
            float4 *dst = reinterpret_cast<float4 *>(a.dv + (size_t)ro * 64 + mm_col<true>(0));
            float4 v = make_float4(acc[p][0], acc[p][1], acc[p][2], acc[p][3]);
            if (a.acc_dv) {
                const float4 o = *dst;
                v.x += o.x; v.y += o.y; v.z += o.z; v.w += o.w;
            }
            *dst = v;
        }
    }
    // dq (rows t, channels i) and dk (rows s, channels i), kept in registers until the
    // shared tiles they replace are free
    float xq[4][4], y1[4][4], y2[4][4];
    zero4x4(xq);
    zero4x4(y1);
    zero4x4(y2);
    mm_acc<false, true, false>(ds, hc, xq);    // sum_j dO[t][j] h_c[i][j]
    mm_acc<false, false, false>(Dm, kh, xq);   // sum_s D[t][s] kh[s][i]
    mm_acc<false, true, false>(vs, dh, y1);    // sum_j v[s][j] dh[i][j]
    mm_acc<true, false, false>(Dm, qh, y2);    // sum_t D[t][s] qh[t][i]
    __syncthreads();   // every product is done: hc and vs now hold dq and dk
    float *dqs = hc, *dks = vs;
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int t = mm_row(p), i = mm_col<false>(r);   // (row t of dq, row s = t of dk)
            dqs[t * kLd + i] = decay_from_start(bs, kz, t, i) * xq[p][r];
            dks[t * kLd + i] = decay_to_end(bs, kz, Bv, Kv, t, i) * y1[p][r] +
                               (fast[i] ? __expf(-bs[t * kLd + i]) * y2[p][r] : 0.f);
        }
    __syncthreads();
    if (any_slow) {   // slow channels' intra-chunk terms of dq and dk
        for (int e = tid; e < kC * kC; e += kThreads) {
            const int t = e >> 6, i = e & 63;
            if (fast[i]) continue;
            float sq = 0.f, sk = 0.f;
            for (int s = 0; s <= t; ++s)   // dq: s <= t
                sq += Dm[t * kLd + s] * ks[s * kLd + i] * decay_ts(bs, kz, t, s, i);
            for (int u = t; u < kC; ++u)   // dk of row t: later rows u >= t
                sk += Dm[u * kLd + t] * qs[u * kLd + i] * decay_ts(bs, kz, u, t, i);
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
        float col[kC];
#pragma unroll
        for (int t = 0; t < kC; ++t) col[t] = xs[t * kLd + tid];
        float s = 0.f;
#pragma unroll
        for (int t = kC - 1; t >= 0; --t) {
            s += col[t];
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
// grid n_seq * nc, 256 threads: dg of the chunk's rows += const + the x totals of the
// later chunks of the sequence.  Channel i = tid % 64; the four quarters of the block
// sum every fourth later chunk (independent loads in flight), then each thread updates
// sixteen rows, every load issued before any store.
__global__ void __launch_bounds__(kThreads) gla_bwd_dg_kernel(const Args a) {
    __shared__ int rows[kC];
    __shared__ float part[4][kC];
    const int tid = threadIdx.x, i = tid & 63, qq = tid >> 6;
    const int seq = (int)(blockIdx.x / a.nc), c = (int)(blockIdx.x % a.nc);
    if (tid < kC) rows[tid] = bwd_row(a, seq, c * kC + tid);
    const float *xc = a.xc + (size_t)seq * a.nc * kC + i;
    float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
    int c2 = c + 1 + qq;
    for (; c2 + 12 < a.nc; c2 += 16) {
        s0 += xc[(size_t)c2 * kC];
        s1 += xc[(size_t)(c2 + 4) * kC];
        s2 += xc[(size_t)(c2 + 8) * kC];
        s3 += xc[(size_t)(c2 + 12) * kC];
    }
    for (; c2 < a.nc; c2 += 4) s0 += xc[(size_t)c2 * kC];
    part[qq][i] = (s0 + s1) + (s2 + s3);
    __syncthreads();
    const float off = a.cst[(size_t)seq * kC + i] + ((part[0][i] + part[1][i]) + (part[2][i] + part[3][i]));
    float v[16];
#pragma unroll
    for (int m = 0; m < 16; ++m) {
        const int ro = rows[qq + 4 * m];
        v[m] = ro >= 0 ? a.dg[(size_t)ro * a.ldk + i] : 0.f;
    }
    issue_fence();
#pragma unroll
    for (int m = 0; m < 16; ++m) {
        const int ro = rows[qq + 4 * m];
        if (ro >= 0) a.dg[(size_t)ro * a.ldk + i] = v[m] + off;
    }
}

}  // namespace bw
}  // namespace gtr
