// gtr_gla.cu -- GTR token-mixer forward pass (key-decay gated linear attention)
// for B200 / sm_100a, behind the C ABI declared in include/gtr_gla.h.
//
// What is computed (GTR news article, tokendh.com, section "线性注意力到底在省什么";
// GTR abstract): per (batch, head) sequence, S_t = diag(exp(g_t)) S_{t-1} + k_t^T v_t
// and o_t = q_t S_t, over one of four scan orders of the patch grid (section
// "单向扫描的致命缺陷，以及GTR怎么补"), chunkwise with 64-token chunks in FP16 with
// FP32 accumulation (section "速度到底快在哪，TensorRT部署做了什么": the heavy work of a
// chunk is parallel, only the chunk-boundary state is passed in order).
//
// Kernel structure (one launch per call):
//   * A thread-block cluster of P CTAs owns one sequence at a time (clusters loop
//     over sequences).  In round r, CTA `rank` processes chunk r*P + rank.
//   * Per chunk, inside one CTA:
//       - q/k/g/v rows are fetched with 16-byte cp.async straight into 128B-swizzled
//         UMMA tiles; the scan direction is applied only in the row addresses.
//       - a = exp(g); inside each 16-token sub-block the inclusive prefix product pi
//         and exclusive suffix product sigma of a, and the sub-block totals T.
//         Every decay factor fed to the tensor cores is a product of a's <= 1,
//         except the diagonal sub-blocks, whose factor pi/T is bounded by exp(8)
//         and falls back to an exact fp32 evaluation beyond that.
//       - tcgen05.mma (fp16 x fp16 -> fp32 in TMEM):
//           dS     = (K * sigma * after)^T V                    (64..128 x 64)
//           scores = (Q * pi * c_J) (K * sigma)^T  per key sub-block J
//           O      = (Q * pi * before) S_prev + tril(scores) V
//   * The chunk-to-chunk state pass S_c = d_c * S_{c-1} + dS_c is the only
//     sequential step.  It runs as an element-sliced scan over the cluster:
//     CTA j reads slice j of every chunk's (d_c, dS_c) from its peers' shared
//     memory (DSMEM), chains it in fp32, and writes S_{c-1} (fp16) straight into
//     the owning CTA's UMMA operand tile.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <mutex>

#include "../../include/gtr_gla.h"
#include "sm100_ptx.cuh"

namespace gtr {

using namespace ptx;

constexpr int kThreads = 256;
constexpr int kChunk = 64;
constexpr int kDV = 64;
constexpr int kSub = 16;              // sub-block length for the decay factorisation
constexpr int kTile = 64 * 128;       // one [64 rows][64 fp16] 128B-swizzled tile
constexpr int kTmemCols = 256;
constexpr int kMaxCluster = 16;
constexpr float kDiagMinTotal = 3.3546262e-4f;  // exp(-8): smallest safe sub-block total
constexpr uint64_t kWaitLimitNs = 200ull * 1000ull * 1000ull;  // 200 ms per bounded wait

enum : unsigned { kErrTimeout = 1u };

__device__ unsigned int g_error_word;

// ------------------------------------------------------------------ smem map
template <int DK>
struct Smem {
    static constexpr int NSUB = DK / 64;
    static constexpr int q = 0;
    static constexpr int k = q + NSUB * kTile;
    static constexpr int g = k + NSUB * kTile;
    static constexpr int v0 = g + NSUB * kTile;
    static constexpr int v1 = v0 + kTile;
    static constexpr int qj = v1 + kTile;                 // packed Q^(J), rows 16J..63
    static constexpr int qj_bytes = NSUB * (64 + 48 + 32 + 16) * 128;
    static constexpr int kbar = qj + qj_bytes;            // K * sigma          [64][DK]
    static constexpr int qint = kbar + NSUB * kTile;      // Q * pi * before    [64][DK]
    static constexpr int kst = qint + NSUB * kTile;       // K * sigma * after  [64][DK]
    static constexpr int p = kst + NSUB * kTile;          // masked scores      [64][64]
    static constexpr int sop = p + kTile;                 // S_prev fp16        [DK][64]
    static constexpr int agg = sop + NSUB * kTile;        // dS fp32            [DK][64]
    static constexpr int dvec = agg + DK * 256;           // d = prod of a      [DK]
    static constexpr int tsh = dvec + DK * 4;             // sub-block totals   [4][DK]
    static constexpr int diag = tsh + 4 * DK * 4;         // exact diag blocks  [4][16][16]
    static constexpr int rowoff = diag + 4 * 16 * 16 * 4; // token rows         [2][64]
    static constexpr int misc = rowoff + 2 * 64 * 4;      // flags, mbarrier, tmem addr
    static constexpr int bytes = misc + 64;
    static constexpr int alloc = bytes + 1024;            // + alignment slack
    // scan staging aliases the Q^(J) region (free between MMA completion and the
    // next round's gating): float4 [P][slice] then float [P][DK]
    static constexpr int stage = qj;
    static constexpr int stage_bytes = qj_bytes;

    static __host__ __device__ constexpr int qj_region(int J) {
        return NSUB * 128 * (J == 0 ? 0 : J == 1 ? 64 : J == 2 ? 112 : 144);
    }
};

// 128B-swizzled [rows][64 fp16] tile: byte offset of (row, col) inside a sub-tile
__device__ __forceinline__ uint32_t sw_off(int row, int col) {
    return (uint32_t)(row * 128 + ((((col >> 3) ^ (row & 7)) & 7) << 4) + ((col & 7) << 1));
}
// fp32 [rows][64] tile swizzled in 16-byte units: byte offset of (row, col4*4)
__device__ __forceinline__ uint32_t agg_off(int row, int col4) {
    return (uint32_t)(row * 256 + (((col4 ^ row) & 15) << 4));
}

__device__ __forceinline__ int scan_to_token(int p, int H, int W, int dir) {
    int y, x;
    if (dir == GTR_L2R) {
        y = p / W; x = p - y * W;
    } else if (dir == GTR_R2L) {
        y = p / W; x = W - 1 - (p - y * W);
    } else if (dir == GTR_T2B) {
        x = p / H; y = p - x * H;
    } else {
        x = p / H; y = H - 1 - (p - x * H);
    }
    return y * W + x;
}

struct Params {
    const __half *q, *k, *v, *g;
    const float *s0;
    __half *out;
    float *sf;
    int B, heads, H, W, N, dir;
    int n_seq, n_chunks;
};

__device__ __forceinline__ void set_error(unsigned e) { atomicOr(&g_error_word, e); }

// ------------------------------------------------------------------ loads
// Issues the cp.async copies of one chunk's q/k/g (into the shared raw tiles)
// and v (into vbuf); rows with rowoff < 0 are zero-filled.
template <int DK>
__device__ __forceinline__ void issue_chunk_loads(const Params &P, uint8_t *sm, const int *rowoff,
                                                  uint32_t vbuf_addr) {
    using L = Smem<DK>;
    constexpr int CPR = DK / 8;              // 16-byte pieces per q/k/g row
    constexpr int QKG = 3 * 64 * CPR;
    constexpr int TOTAL = QKG + 64 * 8;
    const uint32_t base = smem_u32(sm);
    const int tid = threadIdx.x;
#pragma unroll 4
    for (int pid = tid; pid < TOTAL; pid += kThreads) {
        const __half *src;
        uint32_t dst;
        int row;
        if (pid < QKG) {
            const int tsel = pid / (64 * CPR);
            const int rem = pid - tsel * (64 * CPR);
            row = rem / CPR;
            const int cc = rem - row * CPR;
            const __half *tb = tsel == 0 ? P.q : (tsel == 1 ? P.k : P.g);
            const int ro = rowoff[row];
            src = tb + (size_t)(ro < 0 ? 0 : ro) * DK + cc * 8;
            const uint32_t tile = base + (tsel == 0 ? L::q : (tsel == 1 ? L::k : L::g));
            dst = tile + (cc >> 3) * kTile + sw_off(row, (cc & 7) * 8);
            cp_async16(dst, src, ro < 0 ? 0u : 16u);
        } else {
            const int rem = pid - QKG;
            row = rem >> 3;
            const int cc = rem & 7;
            const int ro = rowoff[row];
            src = P.v + (size_t)(ro < 0 ? 0 : ro) * kDV + cc * 8;
            dst = vbuf_addr + sw_off(row, cc * 8);
            cp_async16(dst, src, ro < 0 ? 0u : 16u);
        }
    }
    cp_async_commit();
}

// Token row index ((b*N + n)*heads + h) of each scan position of chunk c, or -1.
__device__ __forceinline__ void fill_rowoff(const Params &P, int seq, int c, int *rowoff) {
    const int t = threadIdx.x;
    if (t < kChunk) {
        int ro = -1;
        if (seq >= 0 && c >= 0) {
            const int p = c * kChunk + t;
            if (p < P.N) {
                const int b = seq / P.heads, h = seq - b * P.heads;
                const int n = scan_to_token(p, P.H, P.W, P.dir);
                ro = (b * P.N + n) * P.heads + h;
            }
        }
        rowoff[t] = ro;
    }
}

// ------------------------------------------------------------------ kernel
template <int DK>
__global__ void __launch_bounds__(kThreads, 1) gla_fwd_kernel(const Params P) {
    using L = Smem<DK>;
    constexpr int ITEMS = DK / 64;        // (channel, sub-block) items per thread in gating
    constexpr int NF4 = DK * kDV / 4;     // float4 elements of the state
    constexpr int MAXM = (NF4 + kThreads - 1) / kThreads;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    const uint32_t rank = cluster_ctarank();
    // cluster size = gridDim.x / number of clusters
    const uint32_t ncl = nclusters_x();
    const int CP = (int)(gridDim.x / ncl);
    const int cl = (int)cluster_id_x();

    float *tsh = reinterpret_cast<float *>(sm + L::tsh);
    float *dvec = reinterpret_cast<float *>(sm + L::dvec);
    float *diagx = reinterpret_cast<float *>(sm + L::diag);
    int *rowoff0 = reinterpret_cast<int *>(sm + L::rowoff);
    int *flags = reinterpret_cast<int *>(sm + L::misc);          // [4] diag fallback flags
    uint64_t *mbar = reinterpret_cast<uint64_t *>(sm + L::misc + 16);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::misc + 32);

    if (warp == 0) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(mbar, 1);
        fence_mbar_init();
    }
    if (tid < 4) flags[tid] = 0;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    uint32_t mma_phase = 0;
    bool timed_out = false;

    // element slice of the state owned by this CTA in the scan
    const int slo = (int)((long)rank * NF4 / CP);
    const int shi = (int)((long)(rank + 1) * NF4 / CP);
    const int nloc = shi - slo;

    int cur = 0;  // rowoff buffer of the current chunk
    int vb = 0;   // v buffer of the current chunk
    // prime the first chunk
    {
        const int seq0 = cl < P.n_seq ? cl : -1;
        const int c0 = (seq0 >= 0 && (int)rank < P.n_chunks) ? (int)rank : -1;
        fill_rowoff(P, seq0, c0, rowoff0);
        __syncthreads();
        if (c0 >= 0) issue_chunk_loads<DK>(P, sm, rowoff0, sbase + L::v0);
    }

    for (int seq = cl; seq < P.n_seq; seq += (int)ncl) {
        const int b = seq / P.heads, h = seq - b * P.heads;
        // running state for this CTA's slice, fp32 registers
        float4 S[MAXM];
#pragma unroll
        for (int m = 0; m < MAXM; ++m) {
            const int el = tid + m * kThreads;
            S[m] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (P.s0 != nullptr && el < nloc)
                S[m] = reinterpret_cast<const float4 *>(P.s0 + (size_t)seq * DK * kDV)[slo + el];
        }
        const int n_rounds = (P.n_chunks + CP - 1) / CP;
        for (int r = 0; r < n_rounds; ++r) {
            const int c = r * CP + (int)rank;
            const bool valid = c < P.n_chunks;
            const int nvalid = min(CP, P.n_chunks - r * CP);
            int *rowoff_cur = rowoff0 + cur * 64;
            int *rowoff_nxt = rowoff0 + (cur ^ 1) * 64;
            const uint32_t vaddr = sbase + (vb ? L::v1 : L::v0);
            const uint32_t vnext = sbase + (vb ? L::v0 : L::v1);

            cp_async_wait_all();
            __syncthreads();

            // ---------------- gating pass 1: a = exp(g), pi, sigma, sub-block totals
            float pa[ITEMS][16];   // pi (inclusive prefix product inside the sub-block)
            float sa[ITEMS][16];   // sigma (exclusive suffix product inside the sub-block)
            if (valid) {
#pragma unroll
                for (int it = 0; it < ITEMS; ++it) {
                    const int item = tid + it * kThreads;
                    const int i = item % DK, I = item / DK;
                    const uint8_t *gt = sm + L::g + (i >> 6) * kTile;
                    float a[16];
#pragma unroll
                    for (int u = 0; u < 16; ++u) {
                        const int t = I * kSub + u;
                        const float gv = __half2float(
                            *reinterpret_cast<const __half *>(gt + sw_off(t, i & 63)));
                        a[u] = __expf(gv);
                    }
                    float run = 1.f;
#pragma unroll
                    for (int u = 0; u < 16; ++u) { run *= a[u]; pa[it][u] = run; }
                    run = 1.f;
#pragma unroll
                    for (int u = 15; u >= 0; --u) { sa[it][u] = run; run *= a[u]; }
                    const float T = pa[it][15];
                    tsh[I * DK + i] = T;
                    if (!(T >= kDiagMinTotal)) atomicOr(&flags[I], 1);
                }
            }
            __syncthreads();

            // ---------------- gating pass 2: UMMA operands (fp16, swizzled)
            if (valid) {
#pragma unroll
                for (int it = 0; it < ITEMS; ++it) {
                    const int item = tid + it * kThreads;
                    const int i = item % DK, I = item / DK;
                    const int ci = i & 63, si = i >> 6;
                    float T[4];
#pragma unroll
                    for (int L2 = 0; L2 < 4; ++L2) T[L2] = tsh[L2 * DK + i];
                    float before = 1.f, after = 1.f;
#pragma unroll
                    for (int L2 = 0; L2 < 4; ++L2) {
                        if (L2 < I) before *= T[L2];
                        if (L2 > I) after *= T[L2];
                    }
                    if (I == 0) dvec[i] = T[0] * T[1] * T[2] * T[3];
                    // coefficient of Q^(J) rows in sub-block I
                    const bool diag_bad = flags[I] != 0;
                    float tI = T[0];
#pragma unroll
                    for (int L2 = 1; L2 < 4; ++L2)
                        if (L2 == I) tI = T[L2];
                    float coef[4];
#pragma unroll
                    for (int J = 0; J < 4; ++J) {
                        float cj = 1.f;
#pragma unroll
                        for (int L2 = 0; L2 < 4; ++L2)
                            if (L2 > J && L2 < I) cj *= T[L2];
                        coef[J] = (J == I) ? (diag_bad ? 0.f : 1.f / tI) : cj;
                    }
                    const uint8_t *qt = sm + L::q + si * kTile;
                    const uint8_t *kt = sm + L::k + si * kTile;
#pragma unroll
                    for (int u = 0; u < 16; ++u) {
                        const int t = I * kSub + u;
                        const uint32_t o = sw_off(t, ci);
                        const float qv = __half2float(*reinterpret_cast<const __half *>(qt + o));
                        const float kv = __half2float(*reinterpret_cast<const __half *>(kt + o));
                        const float qp = qv * pa[it][u];
                        const float ks = kv * sa[it][u];
                        *reinterpret_cast<__half *>(sm + L::qint + si * kTile + o) =
                            __float2half_rn(qp * before);
                        *reinterpret_cast<__half *>(sm + L::kbar + si * kTile + o) =
                            __float2half_rn(ks);
                        *reinterpret_cast<__half *>(sm + L::kst + si * kTile + o) =
                            __float2half_rn(ks * after);
#pragma unroll
                        for (int J = 0; J < 4; ++J) {
                            if (J <= I) {
                                float val = qp * coef[J];
                                if (J == I && !(fabsf(val) <= 60000.f)) {
                                    val = 0.f;
                                    atomicOr(&flags[I], 2);
                                }
                                const int rows_j = 64 - 16 * J;
                                uint8_t *dst = sm + L::qj + L::qj_region(J) + si * rows_j * 128 +
                                               sw_off(t - 16 * J, ci);
                                *reinterpret_cast<__half *>(dst) = __float2half_rn(val);
                            }
                        }
                    }
                }
            }
            // rows of the next chunk (this sequence, or the first round of the next)
            int nseq = seq, nc = c + CP;
            if (nc >= P.n_chunks) {
                nseq = seq + (int)ncl;
                nc = (nseq < P.n_seq && (int)rank < P.n_chunks) ? (int)rank : -1;
                if (nseq >= P.n_seq) nseq = -1;
            }
            fill_rowoff(P, nseq, nc, rowoff_nxt);
            fence_proxy_async_cta();
            __syncthreads();

            // ---------------- exact diagonal sub-blocks where the factorisation is unsafe
            const int anyflag = valid ? (flags[0] | flags[1] | flags[2] | flags[3]) : 0;
            if (anyflag) {
                const uint8_t *qt = sm + L::q, *kt = sm + L::k, *gt = sm + L::g;
                for (int pr = tid; pr < 4 * 256; pr += kThreads) {
                    const int I = pr >> 8, u = (pr >> 4) & 15, w = pr & 15;
                    if (!flags[I] || w > u) continue;
                    const int tu = I * kSub + u, tw = I * kSub + w;
                    float acc = 0.f;
                    for (int i = 0; i < DK; ++i) {
                        const int si = i >> 6, ci = i & 63;
                        float lg = 0.f;
                        for (int rr = tw + 1; rr <= tu; ++rr)
                            lg += __half2float(*reinterpret_cast<const __half *>(
                                gt + si * kTile + sw_off(rr, ci)));
                        const float qv = __half2float(
                            *reinterpret_cast<const __half *>(qt + si * kTile + sw_off(tu, ci)));
                        const float kv = __half2float(
                            *reinterpret_cast<const __half *>(kt + si * kTile + sw_off(tw, ci)));
                        acc += qv * kv * __expf(lg);
                    }
                    diagx[(I * 16 + u) * 16 + w] = acc;
                }
                __syncthreads();
            }

            // prefetch the next chunk (raw q/k/g tiles are no longer needed)
            if (nc >= 0) issue_chunk_loads<DK>(P, sm, rowoff_nxt, vnext);

            // ---------------- MMA 1: dS and the four score column blocks
            if (valid && tid == 0) {
                tc_fence_after();
                {
                    constexpr uint32_t id = idesc_f16_f32(DK, kDV, true, true);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t a = desc_sw128(sbase + L::kst + kk * 2048, kTile, 1024);
                        const uint64_t bd = desc_sw128(vaddr + kk * 2048, kTile, 1024);
                        umma_f16(tmem + 0, a, bd, id, kk > 0 ? 1u : 0u);
                    }
                }
                {
                    constexpr uint32_t id = idesc_f16_f32(64, 16, false, false);
#pragma unroll
                    for (int J = 0; J < 4; ++J) {
                        const int rows_j = 64 - 16 * J;
#pragma unroll
                        for (int kk = 0; kk < DK / 16; ++kk) {
                            const int sub = kk >> 2, koff = (kk & 3) * 32;
                            const uint32_t aa = sbase + L::qj + L::qj_region(J) +
                                                sub * rows_j * 128 - 16 * J * 128 + koff;
                            const uint32_t bb = sbase + L::kbar + sub * kTile + 16 * J * 128 + koff;
                            umma_f16(tmem + 64 + 16 * J, desc_sw128(aa, 16, 1024),
                                     desc_sw128(bb, 16, 1024), id, kk > 0 ? 1u : 0u);
                        }
                    }
                }
                umma_commit(mbar);
            }
            if (valid) {
                if (!mbar_wait_bounded(mbar, mma_phase, kWaitLimitNs)) {
                    timed_out = true;
                    set_error(kErrTimeout);
                }
                mma_phase ^= 1u;
                tc_fence_after();
                if (warp < 4) {
                    // scores -> masked fp16 P (row t = 16*warp + lane)
                    uint32_t rr[64];
                    const uint32_t ta = tmem + ((uint32_t)(32 * warp) << 16) + 64;
                    tmem_ld16(ta + 0, *reinterpret_cast<uint32_t(*)[16]>(&rr[0]));
                    tmem_ld16(ta + 16, *reinterpret_cast<uint32_t(*)[16]>(&rr[16]));
                    tmem_ld16(ta + 32, *reinterpret_cast<uint32_t(*)[16]>(&rr[32]));
                    tmem_ld16(ta + 48, *reinterpret_cast<uint32_t(*)[16]>(&rr[48]));
                    tmem_ld_wait();
                    if (lane < 16) {
                        const int t = 16 * warp + lane;
                        const int It = t >> 4;
                        const bool fb = flags[It] != 0;
#pragma unroll
                        for (int c8 = 0; c8 < 8; ++c8) {
                            uint32_t pk[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                float x[2];
#pragma unroll
                                for (int z = 0; z < 2; ++z) {
                                    const int s = c8 * 8 + e * 2 + z;
                                    float val = __uint_as_float(rr[s]);
                                    if (fb && (s >> 4) == It) val = diagx[(It * 16 + (t & 15)) * 16 + (s & 15)];
                                    x[z] = s <= t ? val : 0.f;
                                }
                                pk[e] = pack_half2(x[0], x[1]);
                            }
                            *reinterpret_cast<uint4 *>(sm + L::p + t * 128 + (((c8 ^ (t & 7)) & 7) << 4)) =
                                make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        }
                    }
                } else {
                    // dS -> fp32 aggregate tile for the cluster scan
                    const int sub = warp - 4;
                    uint32_t rr[64];
                    const uint32_t ta = tmem + ((uint32_t)(32 * sub) << 16);
                    tmem_ld16(ta + 0, *reinterpret_cast<uint32_t(*)[16]>(&rr[0]));
                    tmem_ld16(ta + 16, *reinterpret_cast<uint32_t(*)[16]>(&rr[16]));
                    tmem_ld16(ta + 32, *reinterpret_cast<uint32_t(*)[16]>(&rr[32]));
                    tmem_ld16(ta + 48, *reinterpret_cast<uint32_t(*)[16]>(&rr[48]));
                    tmem_ld_wait();
                    const bool has_row = DK == 128 || lane < 16;
                    if (has_row) {
                        const int i = DK == 128 ? 32 * sub + lane : 16 * sub + lane;
#pragma unroll
                        for (int c4 = 0; c4 < 16; ++c4)
                            *reinterpret_cast<float4 *>(sm + L::agg + agg_off(i, c4)) =
                                make_float4(__uint_as_float(rr[4 * c4]), __uint_as_float(rr[4 * c4 + 1]),
                                            __uint_as_float(rr[4 * c4 + 2]), __uint_as_float(rr[4 * c4 + 3]));
                    }
                }
            }
            fence_proxy_async_cta();
            tc_fence_before();
            cluster_sync();   // every chunk's (d, dS) of this round is visible cluster-wide
            if (tid < 4) flags[tid] = 0;  // every reader of this round's flags has passed the barrier

            // ---------------- state pass, step A: stage peers' (d, dS) slices locally
            float4 *stg = reinterpret_cast<float4 *>(sm + L::stage);
            float *stgd = reinterpret_cast<float *>(sm + L::stage + (size_t)CP * nloc * 16);
            for (int x = tid; x < nvalid * nloc; x += kThreads) {
                const int j = x / nloc, el = x - j * nloc;
                const int e = slo + el, i = e >> 4, c4 = e & 15;
                stg[x] = ld_dsmem_f4(mapa(sbase + L::agg + agg_off(i, c4), (uint32_t)j));
            }
            {
                const int ilo = slo >> 4, ihi = (shi + 15) >> 4;   // rows touched by the slice
                const int nr = ihi - ilo;
                for (int x = tid; x < nvalid * nr; x += kThreads) {
                    const int j = x / nr, ii = x - j * nr;
                    stgd[j * DK + ilo + ii] =
                        ld_dsmem_f32(mapa(sbase + L::dvec + (ilo + ii) * 4, (uint32_t)j));
                }
            }
            __syncthreads();
            // ---------------- step B: chain the slice through the round's chunks
#pragma unroll
            for (int m = 0; m < MAXM; ++m) {
                const int el = tid + m * kThreads;
                if (el < nloc) {
                    const int e = slo + el, i = e >> 4, c4 = e & 15;
                    const uint32_t soff = sbase + L::sop + sw_off(i, 4 * c4);
                    for (int j = 0; j < nvalid; ++j) {
                        st_dsmem_v2(mapa(soff, (uint32_t)j), pack_half2(S[m].x, S[m].y),
                                    pack_half2(S[m].z, S[m].w));
                        const float4 a4 = stg[j * nloc + el];
                        const float d = stgd[j * DK + i];
                        S[m].x = fmaf(d, S[m].x, a4.x);
                        S[m].y = fmaf(d, S[m].y, a4.y);
                        S[m].z = fmaf(d, S[m].z, a4.z);
                        S[m].w = fmaf(d, S[m].w, a4.w);
                    }
                }
            }
            fence_proxy_async_cluster();
            cluster_sync();   // every S_prev tile of this round is written

            // ---------------- MMA 2: O = Qint S_prev + tril(scores) V
            if (valid && tid == 0) {
                tc_fence_after();
                constexpr uint32_t id = idesc_f16_f32(64, kDV, false, true);
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk) {
                    const uint32_t aa = sbase + L::qint + (kk >> 2) * kTile + (kk & 3) * 32;
                    const uint32_t bb = sbase + L::sop + kk * 2048;
                    umma_f16(tmem + 128, desc_sw128(aa, 16, 1024), desc_sw128(bb, kTile, 1024), id,
                             kk > 0 ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint32_t aa = sbase + L::p + kk * 32;
                    const uint32_t bb = vaddr + kk * 2048;
                    umma_f16(tmem + 128, desc_sw128(aa, 16, 1024), desc_sw128(bb, kTile, 1024), id, 1u);
                }
                umma_commit(mbar);
            }
            if (valid) {
                if (!mbar_wait_bounded(mbar, mma_phase, kWaitLimitNs)) {
                    timed_out = true;
                    set_error(kErrTimeout);
                }
                mma_phase ^= 1u;
                tc_fence_after();
                if (warp < 4) {
                    uint32_t rr[64];
                    const uint32_t ta = tmem + ((uint32_t)(32 * warp) << 16) + 128;
                    tmem_ld16(ta + 0, *reinterpret_cast<uint32_t(*)[16]>(&rr[0]));
                    tmem_ld16(ta + 16, *reinterpret_cast<uint32_t(*)[16]>(&rr[16]));
                    tmem_ld16(ta + 32, *reinterpret_cast<uint32_t(*)[16]>(&rr[32]));
                    tmem_ld16(ta + 48, *reinterpret_cast<uint32_t(*)[16]>(&rr[48]));
                    tmem_ld_wait();
                    if (lane < 16) {
                        const int t = 16 * warp + lane;
                        const int ro = rowoff_cur[t];
                        if (ro >= 0) {
                            uint4 *dst = reinterpret_cast<uint4 *>(P.out + (size_t)ro * kDV);
#pragma unroll
                            for (int c8 = 0; c8 < 8; ++c8)
                                dst[c8] = make_uint4(
                                    pack_half2(__uint_as_float(rr[8 * c8 + 0]), __uint_as_float(rr[8 * c8 + 1])),
                                    pack_half2(__uint_as_float(rr[8 * c8 + 2]), __uint_as_float(rr[8 * c8 + 3])),
                                    pack_half2(__uint_as_float(rr[8 * c8 + 4]), __uint_as_float(rr[8 * c8 + 5])),
                                    pack_half2(__uint_as_float(rr[8 * c8 + 6]), __uint_as_float(rr[8 * c8 + 7])));
                        }
                    }
                }
            }
            tc_fence_before();
            cur ^= 1;
            vb ^= 1;
        }
        // final state of this sequence
        if (P.sf != nullptr) {
#pragma unroll
            for (int m = 0; m < MAXM; ++m) {
                const int el = tid + m * kThreads;
                if (el < nloc)
                    reinterpret_cast<float4 *>(P.sf + (size_t)seq * DK * kDV)[slo + el] = S[m];
            }
        }
        (void)b;
        (void)h;
    }

    cp_async_wait_all();
    __syncthreads();
    if (timed_out) {
        // let any MMA still in flight finish before giving TMEM back
        mbar_wait_bounded(mbar, mma_phase ^ 1u, kWaitLimitNs);
    }
    cluster_sync();   // no CTA leaves while a peer may still touch its shared memory
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------------ host
struct Plan {
    int cluster, clusters, smem;
};

static int g_num_sms = 0;
static std::mutex g_mu;

static int num_sms() {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_num_sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        g_num_sms = n;
    }
    return g_num_sms;
}

static Plan make_plan(long n_seq, long n_chunks, int dk, int sms) {
    Plan p{};
    p.smem = dk == 64 ? Smem<64>::alloc : Smem<128>::alloc;
    long cp = n_seq > 0 ? sms / n_seq : 1;
    if (n_chunks == 0 || cp < 1) cp = 1;
    if (cp > kMaxCluster) cp = kMaxCluster;
    if (n_chunks > 0 && cp > n_chunks) cp = n_chunks;
    if (cp < 1) cp = 1;
    // the scan staging (P slices of dS plus P rows of d) must fit its region
    const int nf4 = dk * kDV / 4;
    const int stage_bytes = dk == 64 ? Smem<64>::stage_bytes : Smem<128>::stage_bytes;
    while (cp > 1 && (long)(nf4 + cp) * 16 + (long)cp * dk * 4 > stage_bytes) --cp;
    p.cluster = (int)cp;
    long ncl = sms / cp;
    if (ncl > n_seq) ncl = n_seq;
    if (ncl < 1) ncl = 1;
    p.clusters = (int)ncl;
    return p;
}

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <int DK>
static cudaError_t launch(const Params &prm, const Plan &pl, cudaStream_t stream) {
    auto kern = gla_fwd_kernel<DK>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem);
    if (e != cudaSuccess) return e;
    if (pl.cluster > 8) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(pl.cluster * pl.clusters), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = (size_t)pl.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)pl.cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, prm);
}

}  // namespace gtr

using namespace gtr;

static gtr_status_t check_args(const void *q, const void *k, const void *v, const void *g,
                               int B, int heads, int H, int W, int dk, int dv, int dir,
                               int chunk, const float *s0, const void *out, const float *sf) {
    if (B <= 0 || heads <= 0 || H < 0 || W < 0 || dk <= 0 || dv <= 0) return GTR_ERR_INVALID_ARG;
    const bool empty = (long long)H * W == 0;   // an empty grid reads and writes no token
    if (!empty && (!q || !k || !v || !g || !out)) return GTR_ERR_INVALID_ARG;
    if (dir < 0 || dir > 3) return GTR_ERR_INVALID_ARG;
    if (chunk <= 0) return GTR_ERR_INVALID_ARG;
    if (chunk != kChunk) return GTR_ERR_UNSUPPORTED;
    if ((dk != 64 && dk != 128) || dv != kDV) return GTR_ERR_UNSUPPORTED;
    if ((!empty && (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) ||
                    !aligned16(out))) ||
        (s0 && !aligned16(s0)) || (sf && !aligned16(sf)))
        return GTR_ERR_INVALID_ARG;
    const long long N = (long long)H * W;
    const long long rows = (long long)B * N * heads;
    if (N > 0x7fffffffLL || rows * (long long)dk > 0x7fffffffLL || rows * dv > 0x7fffffffLL)
        return GTR_ERR_INVALID_ARG;
    // out may not overlap any input
    const long long qbytes = rows * dk * 2, vbytes = rows * dv * 2;
    auto overlap = [](const void *a, long long na, const void *b, long long nb) {
        const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
        return na > 0 && nb > 0 && x < y + (uintptr_t)nb && y < x + (uintptr_t)na;
    };
    if (overlap(out, vbytes, q, qbytes) || overlap(out, vbytes, k, qbytes) ||
        overlap(out, vbytes, g, qbytes) || overlap(out, vbytes, v, vbytes))
        return GTR_ERR_INVALID_ARG;
    return GTR_OK;
}

extern "C" gtr_status_t gtr_gla_fwd(const gtr_half_t *q, const gtr_half_t *k,
                                    const gtr_half_t *v, const gtr_half_t *g, int B, int heads,
                                    int Hgrid, int Wgrid, int dk, int dv, int direction, int chunk,
                                    const float *init_state, gtr_half_t *out, float *final_state,
                                    void *stream) {
    const gtr_status_t st = check_args(q, k, v, g, B, heads, Hgrid, Wgrid, dk, dv, direction,
                                       chunk, init_state, out, final_state);
    if (st != GTR_OK) return st;
    Params prm{};
    prm.q = reinterpret_cast<const __half *>(q);
    prm.k = reinterpret_cast<const __half *>(k);
    prm.v = reinterpret_cast<const __half *>(v);
    prm.g = reinterpret_cast<const __half *>(g);
    prm.s0 = init_state;
    prm.out = reinterpret_cast<__half *>(out);
    prm.sf = final_state;
    prm.B = B;
    prm.heads = heads;
    prm.H = Hgrid;
    prm.W = Wgrid;
    prm.N = Hgrid * Wgrid;
    prm.dir = direction;
    prm.n_seq = B * heads;
    prm.n_chunks = (prm.N + kChunk - 1) / kChunk;
    const Plan pl = make_plan(prm.n_seq, prm.n_chunks, dk, num_sms());
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const cudaError_t e = dk == 64 ? launch<64>(prm, pl, s) : launch<128>(prm, pl, s);
    return e == cudaSuccess ? GTR_OK : GTR_ERR_CUDA;
}

extern "C" gtr_status_t gtr_gla_device_status(void *stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) {
        cudaGetLastError();
        return GTR_ERR_CUDA;
    }
    unsigned word = 0;
    if (cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word)) != cudaSuccess) return GTR_ERR_CUDA;
    if (word != 0) {
        const unsigned zero = 0;
        cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero));
        return GTR_ERR_TIMEOUT;
    }
    return GTR_OK;
}

extern "C" const char *gtr_status_str(gtr_status_t s) {
    switch (s) {
    case GTR_OK: return "ok";
    case GTR_ERR_INVALID_ARG: return "invalid argument";
    case GTR_ERR_UNSUPPORTED: return "unsupported configuration";
    case GTR_ERR_CUDA: return "CUDA error";
    case GTR_ERR_TIMEOUT: return "device-side wait timed out";
    }
    return "unknown status";
}

extern "C" gtr_status_t gtr_gla_plan(int B, int heads, int Hgrid, int Wgrid, int dk, int dv,
                                     int *cluster_size, int *num_clusters, int *smem_bytes) {
    if (B <= 0 || heads <= 0 || Hgrid < 0 || Wgrid < 0) return GTR_ERR_INVALID_ARG;
    if ((dk != 64 && dk != 128) || dv != kDV) return GTR_ERR_UNSUPPORTED;
    const long long N = (long long)Hgrid * Wgrid;
    const Plan pl = make_plan((long)B * heads, (long)((N + kChunk - 1) / kChunk), dk, num_sms());
    if (cluster_size) *cluster_size = pl.cluster;
    if (num_clusters) *num_clusters = pl.clusters;
    if (smem_bytes) *smem_bytes = pl.smem;
    return GTR_OK;
}

extern "C" const char *gtr_gla_version(void) { return "0.1.0"; }
