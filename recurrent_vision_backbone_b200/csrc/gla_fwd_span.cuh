// gla_fwd_span.cuh -- span-parallel GTR token-mixer forward kernel for dk = dv = 64
// (included by gtr_gla.cu, which holds the shared helpers and the C ABI).
//
// Decomposition.  Each (batch, head) sequence is cut into P contiguous spans of
// chunks; one CTA owns one span (persistent CTAs loop over sequences).  Inside a
// span the chunk-to-chunk state pass (GTR news article, section
// "速度到底快在哪，TensorRT部署做了什么": only the chunk-boundary state is passed in order)
// is purely local, so no per-chunk traffic crosses CTAs:
//
//   phase 1  stream the span's chunks from a zero state (span 0: from S0), as a
//            pipeline over two operand buffers:
//              loaders (warps 12 ..) cp.async of q, k, g rows into staging and of v
//                                 straight into its swizzled operand tile, two
//                                 chunks ahead, as the buffers free up;
//              group A (warps 0-7) gating of chunk c (Qint = q P, K~ = k / P, ...),
//                                 then S <- d * S + dS of chunk c-1 from TMEM (its
//                                 fp16 copy is S_prev of chunk c);
//              group B (warps 8-11) once chunk c is gated, MMA 1(c) = (dS, scores)
//                                 (one elected lane: MMA 2(c-1), which consumed the
//                                 scores' TMEM columns, is complete by then), then the
//                                 scores of chunk c from TMEM into the causal fp16
//                                 P tile, written back to TMEM, MMA 2(c) = Qint S_prev
//                                 + P V (P as the TMEM A operand), output stores
//                                 (spans of at most kShortSpan chunks, span 0 included,
//                                 keep every output in TMEM until phase 4);
//   phase 2  the span's last state update publishes its aggregate (state reached
//            from zero, product of the decays) to the workspace (in short spans group
//            B does that update, right after its last MMA 2).
//   phase 3  look back: fold the aggregates of the earlier spans into S_in, the true
//            state entering this span (short spans: each aggregate is copied into
//            shared memory as soon as its flag is seen, and the fold writes the fp16
//            operand of phase 4 directly).
//   phase 4  correct the outputs for the missing S_in term.  For a chunk c starting
//            D_c (per key channel, product of the decays since the span start) into the
//            span, the term is (Q * P) diag(D_c) S_in.  The first kHold chunks keep
//            their fp32 outputs in TMEM and get the exact term added by one MMA each;
//            later chunks get it by re-reading q, g and o, unless a bound shows the term
//            is below 2^-16 of the chunk's largest output (the decays make it vanish
//            after a few chunks for the gates on the pages' workloads).
//   phase 5  the last span writes the final state  D_span * S_in + S_local.
//
// All spans of a sequence are co-resident (cooperative launch), so the look-back
// waits always end; every wait is bounded anyway.
#pragma once

namespace gtr {
namespace sp {

constexpr int kThreadsA = 256;              // warps 0-7
constexpr int kThreadsB = 128;              // warps 8-11
// Loader warps (12 ..): two for long spans; four for spans of at most
// kShortSpan chunks, which are latency-bound and gain from issuing a chunk's loads
// faster (long spans lose: more warps share the schedulers with the compute groups)
template <int NL>
__host__ __device__ constexpr int span_threads() { return kThreadsA + kThreadsB + 32 * NL; }
constexpr int kShortSpan = 4;
constexpr int kDK = 64;
constexpr int kHold = 4;                    // chunks per span whose outputs wait in TMEM
static_assert(kShortSpan <= kHold, "a short span holds every chunk's output in TMEM");
constexpr int kMaxSpan = 32;                // chunks of a span with recorded decays
constexpr uint32_t kBarA = 1, kBarB = 2;    // named barriers; 3..5: phase-4 epilogue teams
constexpr uint32_t kBarPro = 6;             // groups A and B: sequence prologue
constexpr int kAggFloats = kDK * kDV + kDK; // state + decay product
// TMEM columns: dS of MMA 1 (two buffers), scores of MMA 1, MMA 2 work block, the
// held chunks' output blocks
constexpr uint32_t kColDS = 0, kColScores = 128, kColWork = 192, kColHold = 256;
constexpr int kSpanTmemCols = 512;

// ------------------------------------------------------------------ smem map
struct L {
    static constexpr int stg_bytes = 3 * kTile;         // raw rows q, k, g [64][128 B]
    static constexpr int stg = 0;                       // x2 buffers
    static constexpr int vop = stg + 2 * stg_bytes;     // V swizzled (loaded directly), x3
    static constexpr int qint = vop + 3 * kTile;        // Q * P, x2
    static constexpr int kt = qint + 2 * kTile;         // K / P or K * sigma * after, x2
    static constexpr int p = kt + 2 * kTile;            // masked scores, then output staging
    static constexpr int qj = p + kTile;                // packed Q^(J) (sub-block path)
    static constexpr int qj_bytes = (64 + 48 + 32 + 16) * 128;
    static constexpr int kbar = qj + qj_bytes;          // K * sigma (sub-block path)
    static constexpr int sop = kbar + kTile;            // S_prev fp16, x2
    static constexpr int sst = sop + 2 * kTile;         // running state fp32 [64][64] swizzled
    static constexpr int ring = sst + 64 * 256;         // Qint * D_c of the held chunks
    static constexpr int dcum = ring + kHold * kTile;   // D_c, c = 0 .. kMaxSpan [kMaxSpan+1][64]
    static constexpr int dloc = dcum + (kMaxSpan + 1) * 256;   // chunk decay d [2][64]
    static constexpr int htot = dloc + 2 * 256;         // half-block totals [8][64]
    static constexpr int diag = htot + 8 * 64 * 4;      // exact diagonal blocks [2][4][16][16]
    static constexpr int rowb = diag + 2 * 4 * 16 * 16 * 4; // token rows [3 teams][64]
    static constexpr int cmeta = rowb + 3 * 64 * 4;     // per chunk: max|q|, max|o| [kMaxSpan][2]
    static constexpr int skipf = cmeta + kMaxSpan * 8;  // per chunk: correction negligible
    static constexpr int rmax = skipf + kMaxSpan * 4;   // row maxima of |S_in| [64]
    static constexpr int ltab = rmax + 256;             // loaders' token rows [64]
    static constexpr int misc = ltab + 256;             // per parity (64 B): flags[4] qmax[4] kmax
    static constexpr int bars = misc + 128;
    static constexpr int bytes = bars + 24 * 8;
    static constexpr int alloc = bytes + 1024;
    // after phase 1 the K~ tiles hold S_in (fp32 [64][64], swizzled)
    static constexpr int sin = kt;

    static __host__ __device__ constexpr int qj_region(int J) {
        return 128 * (J == 0 ? 0 : J == 1 ? 64 : J == 2 ? 112 : 144);
    }
};
static_assert(L::alloc <= 227 * 1024, "shared memory budget");

enum {
    B_STGF = 0,   // [2] staging (+ V tile) landed: 64 loader arrivals
    B_STGE = 2,   // [2] group A done with the staging buffer
    B_MMA1 = 19,  // [2] MMA 1 of a chunk of this parity complete (waited by groups A and B)
    B_OPSF = 6,   // [2] S_prev of a chunk ready for its MMA 2
    B_OPSE = 8,   // [2] MMA 2 done with Qint, S_prev of a buffer (tcgen05.commit)
    B_MMA2 = 10,
    B_FIX = 11,   // correction MMAs complete
    B_TMEM = 13,  // (uint32_t) TMEM base
    B_VE = 14,    // [3] MMA 2 done with a V tile (tcgen05.commit)
    B_GATE = 17   // [2] group A's gating of a chunk done (operands, flags, diagonal blocks)
};

// Workspace protocol.  Every flag is zero when a launch starts.  Span k of a
// sequence publishes its aggregate by storing (release) the number of its readers,
// P - 1 - k, into its flag; each later span waits (acquire) for a non-zero flag and
// then takes one off it (a reduction, nothing waits on it).  The last reader
// leaves the flag at zero, so the workspace is clean again when the launch ends and
// any shape may use it next.  The flags sit at a fixed offset whatever the shape.
struct Work {
    int P;        // spans per sequence
    int Lc;       // chunks per span (the last span may be shorter)
    float *ws;    // [n_seq][P][kAggFloats] aggregates
    unsigned *flags;   // [n_seq][P] publish flags (readers still to come), kFlagStride apart
    float inv_tau;     // the gate's 1 / tau (kernels that read z in place of g)
};
// One 128-byte line per flag: every later span of a sequence polls its predecessors'
// flags, and packed flags made a few L2 lines the hot spot of all those polls (a
// probe on the B200 measured the visibility tail at 3.5 us packed, 1.8 us padded).
constexpr int kFlagStride = 32;

__device__ __forceinline__ uint64_t *bar(uint8_t *sm, int i) {
    return reinterpret_cast<uint64_t *>(sm + L::bars) + i;
}
// Bounded wait; after the first timeout a thread stops waiting (its results are
// garbage then, but the kernel still ends and the error word reports it).
__device__ __forceinline__ void wait_l(uint64_t *b, uint32_t parity, bool &to) {
    if (to) return;
    if (!mbar_wait_bounded(b, parity, kWaitLimitNs)) {
        to = true;
        set_error(kErrTimeout);
    }
}
// Waits for phase `k` of a barrier whose phases complete in order, given the count
// `seen` of phases this thread has already observed (never more than one phase can
// be ahead of the waiter for the barriers this is used on).
__device__ __forceinline__ void wait_phase(uint64_t *b, uint32_t &seen, uint32_t k, bool &to) {
    while (seen <= k) {
        wait_l(b, seen & 1u, to);
        ++seen;
    }
}

// Loader warp `lw` (of NL): its share of chunk c's 64 rows of q, k, g into
// staging buffer `b` (row t at byte t * 128, unswizzled) and of v into the swizzled
// operand tile vop[vb], with 16-byte cp.async, eight lanes per 128-byte row so that
// one warp instruction moves four whole rows: rows 4 (NL i + lw) + lane / 8.
// Rows past the grid are zero-filled.
template <int NL>
__device__ __forceinline__ void load_chunk(const Params &P, uint8_t *sm, int seq, int c, int b,
                                           int vb, int lane, int lw) {
    constexpr int kRows = 64 / NL;   // rows of this warp
    const uint32_t st = smem_u32(sm + L::stg + b * L::stg_bytes);
    const uint32_t vo = smem_u32(sm + L::vop + vb * kTile);
    int *rowtab = reinterpret_cast<int *>(sm + L::ltab) + kRows * lw;
    const int bb = seq / P.heads, h = seq - bb * P.heads;
    __syncwarp();   // every lane is done with the previous chunk's table
    for (int r = lane; r < kRows; r += 32) {
        const int t = 4 * (NL * (r >> 2) + lw) + (r & 3), p = c * kChunk + t;
        rowtab[r] = p < P.N ? (bb * P.N + scan_to_token(p, P.H, P.W, P.dir)) * P.heads + h : -1;
    }
    __syncwarp();
    const int sub = lane >> 3, pc = lane & 7;
#pragma unroll 4
    for (int i = 0; i < kRows / 4; ++i) {
        const int t = 4 * (NL * i + lw) + sub;
        const int ro = rowtab[4 * i + sub];
        const uint32_t nb = ro >= 0 ? 16u : 0u;
        const size_t rr = (size_t)(ro >= 0 ? ro : 0);
        const size_t off = rr * P.ldk + 8 * pc;   // q, k, g rows (pitch: dk of the call)
        const uint32_t d = st + t * 128 + 16 * pc;
        cp_async16(d, P.q + off, nb);
        cp_async16(d + kTile, P.k + off, nb);
        cp_async16(d + 2 * kTile, P.g + off, nb);
        cp_async16(vo + sw_off(t, 8 * pc), P.v + rr * P.ldv + 8 * pc, nb);
    }
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_gpu(unsigned *p, unsigned v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void red_dec_gpu(unsigned *p) {   // *p -= 1, relaxed, no result
    asm volatile("red.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(0xffffffffu) : "memory");
}
// Waits (acquire) until *f is non-zero, for at most limit_ns; false if the limit ran out.
__device__ __forceinline__ bool flag_wait_bounded(const unsigned *f, uint64_t limit_ns) {
    if (ld_acquire_gpu(f) != 0u) return true;
    const long long t0 = cycles(), lim = cycles_of_ns(limit_ns);
    while (ld_acquire_gpu(f) == 0u) {
        if (cycles() - t0 > lim) return false;
        __nanosleep(32);
    }
    return true;
}

// Epilogue of one 64x64 fp32 accumulator at TMEM column `col` by a team of four
// consecutive warps (warp w reads TMEM lanes 32 (w % 4) ..; tb = thread in the team,
// named barrier `bar_id`): adds `addend` rows from an unswizzled fp16 staging tile if
// non-null, converts to fp16 through the staging tile `os`, stores at the token rows
// in `rowb` (with P.acc and no addend: adds to the rows stored there); returns this
// thread's max |value|.
__device__ __forceinline__ float store_chunk_out(const Params &P, uint32_t tmem, uint32_t col,
                                                 int bw, int lane, int tb, const uint8_t *addend,
                                                 uint32_t bar_id, uint8_t *os, const int *rowb) {
    uint32_t r0[16], r1[16];
    const uint32_t ta = tmem + ((uint32_t)(32 * bw) << 16) + col;
    tmem_ld_16x256b_x4(ta, r0);
    tmem_ld_16x256b_x4(ta + 32, r1);
    tmem_ld_wait();
    const int row0 = 16 * bw + (lane >> 2);
    const int col0 = 2 * (lane & 3);
    float mx = 0.f;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int row = row0 + 8 * hh;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int col = col0 + 8 * cc + 32 * half;
                const uint32_t *rr = half ? r1 : r0;
                float x0 = __uint_as_float(rr[4 * cc + 2 * hh]);
                float x1 = __uint_as_float(rr[4 * cc + 2 * hh + 1]);
                if (addend) {
                    const float2 a = ld_h2(addend + row * 128 + 2 * col);
                    x0 += a.x;
                    x1 += a.y;
                }
                mx = fmaxf(mx, fmaxf(fabsf(x0), fabsf(x1)));
                st_h2(os + sw_off(row, col), x0, x1);
            }
        }
    tc_fence_before();
    named_sync(bar_id, 128);
    // (a correction passes the stored rows as `addend`: the sum is then stored as is)
    if (!P.acc || addend != nullptr) {
#pragma unroll
        for (int x = tb; x < 64 * 8; x += 128) {
            const int row = x >> 3, c8 = x & 7;
            const int ro = rowb[row];
            if (ro >= 0)
                *reinterpret_cast<uint4 *>(P.out + (size_t)ro * P.ldv + 8 * c8) =
                    *reinterpret_cast<const uint4 *>(os + sw_off(row, 8 * c8));
        }
    } else {
        // the second key-channel half of a dk = 128 call: add to what the first half
        // stored (the launches are ordered on the stream); the sum is range-checked
        uint4 cur[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {   // the loads first, so that their latencies overlap
            const int x = tb + 128 * i, row = x >> 3, c8 = x & 7;
            const int ro = rowb[row];
            cur[i] = *reinterpret_cast<const uint4 *>(P.out + (size_t)(ro >= 0 ? ro : 0) * P.ldv + 8 * c8);
        }
        __half2 m2 = __float2half2_rn(0.f);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int x = tb + 128 * i, row = x >> 3, c8 = x & 7;
            const int ro = rowb[row];
            const uint4 a = *reinterpret_cast<const uint4 *>(os + sw_off(row, 8 * c8));
            const uint32_t cw[4] = {cur[i].x, cur[i].y, cur[i].z, cur[i].w}, aw[4] = {a.x, a.y, a.z, a.w};
            uint32_t vw[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const __half2 v = __hadd2(*reinterpret_cast<const __half2 *>(&cw[m]),
                                          *reinterpret_cast<const __half2 *>(&aw[m]));
                vw[m] = *reinterpret_cast<const uint32_t *>(&v);
                if (ro >= 0) m2 = __hmax2_nan(m2, __habs2(v));
            }
            if (ro >= 0)
                *reinterpret_cast<uint4 *>(P.out + (size_t)ro * P.ldv + 8 * c8) = make_uint4(vw[0], vw[1], vw[2], vw[3]);
        }
        const float ml = __low2float(m2), mh = __high2float(m2);
        mx = (ml != ml || mh != mh) ? ml + mh : fmaxf(mx, fmaxf(ml, mh));
    }
    named_sync(bar_id, 128);
    range_check(mx);   // the fp16 outputs
    return mx;
}

__device__ __forceinline__ void fill_rows(const Params &P, int seq, int c, int *rowb, int tb) {
    if (tb < 64) {
        const int p = c * kChunk + tb;
        int ro = -1;
        if (p < P.N) {
            const int bb = seq / P.heads, hh = seq - bb * P.heads;
            ro = (bb * P.N + scan_to_token(p, P.H, P.W, P.dir)) * P.heads + hh;
        }
        rowb[tb] = ro;
    }
}

// Per-parity scratch of group A (64 bytes): flags[4] (sub-block uses the exact
// diagonal), qmax[4] (max |q| per sub-block), kmax (max |k|), slow.
__device__ __forceinline__ int *misc_flags(uint8_t *sm, int b) {
    return reinterpret_cast<int *>(sm + L::misc + 64 * b);
}
__device__ __forceinline__ unsigned *misc_qmax(uint8_t *sm, int b) {
    return reinterpret_cast<unsigned *>(sm + L::misc + 64 * b + 16);
}
__device__ __forceinline__ unsigned *misc_kmax(uint8_t *sm, int b) {
    return reinterpret_cast<unsigned *>(sm + L::misc + 64 * b + 32);
}
__device__ __forceinline__ int *misc_slow(uint8_t *sm, int b) {   // chunk took the sub-block path
    return reinterpret_cast<int *>(sm + L::misc + 64 * b + 36);
}

// Group A (threads 0..255): gating of chunk ci of the span from staging buffer b.
// Writes Qint -> qint[b], K~ -> kt[b] (sub-block path: also Q^(J) -> qj, K sigma ->
// kbar, exact diagonal blocks -> diag[b]), Qint * D_ci -> ring[ci] for a held chunk,
// the chunk decay d -> dloc[b] and D_{ci+1} -> dcum, then signals GATE[b].  The
// sub-block path first waits for MMA 1 of chunk ci-1 (phase index `m1_prev`; it may
// still read qj / kbar).  Returns true on the sub-block path.
template <bool kZ>
__device__ __forceinline__ bool gate_chunk(const Params &P, uint8_t *sm, int ci, int b, int nrows,
                                           bool held, uint32_t &m1_seen, uint32_t m1_prev, bool &to,
                                           float inv_tau) {
    // (m1_seen / m1_prev: phase count and index of MMA 1 of chunk ci-1 on MMA1[b ^ 1])
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gI = warp >> 1, ghf = warp & 1, gt0 = 16 * gI + 8 * ghf, gh = 2 * gI + ghf;
    float *htot = reinterpret_cast<float *>(sm + L::htot);
    float *diagx = reinterpret_cast<float *>(sm + L::diag) + b * 1024;
    float *dcum = reinterpret_cast<float *>(sm + L::dcum);
    const uint8_t *st = sm + L::stg + b * L::stg_bytes;
    uint8_t *qo = sm + L::qint + b * kTile;
    uint8_t *ko = sm + L::kt + b * kTile;
    uint8_t *qr = sm + L::ring + (held ? ci : 0) * kTile;
    int *flags = misc_flags(sm, b);
    unsigned *qmax = misc_qmax(sm, b);
    unsigned *kmax = misc_kmax(sm, b);
    // group B read this parity's flags and diagonal blocks (chunk ci-2) before its MMA 2,
    // whose completion released this buffer
    if (tid < 4) flags[tid] = 0;
    // ---------- pass 1: a = exp(g), half-block prefix / suffix products and totals
    float pl[8][2], sl[8][2];
    __half2 qh[8], kh[8];
    {
        __half2 qm2 = __float2half2_rn(0.f), km2 = __float2half2_rn(0.f);
        float a0[8], a1[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const uint32_t o = (gt0 + u) * 128 + 4 * lane;
            float2 gv = ld_h2(st + 2 * kTile + o);
            if constexpr (kZ)   // rows past the grid keep g = 0 (their z is the zero fill)
                gv = gt0 + u < nrows ? gate2<kZ>(gv, inv_tau) : make_float2(0.f, 0.f);
            qh[u] = *reinterpret_cast<const __half2 *>(st + o);
            kh[u] = *reinterpret_cast<const __half2 *>(st + kTile + o);
            a0[u] = exp_f(gv.x);
            a1[u] = exp_f(gv.y);
            qm2 = __hmax2(qm2, __habs2(qh[u]));
            km2 = __hmax2(km2, __habs2(kh[u]));
        }
        float r0 = 1.f, r1 = 1.f;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            r0 *= a0[u];
            r1 *= a1[u];
            pl[u][0] = r0;
            pl[u][1] = r1;
        }
        r0 = 1.f;
        r1 = 1.f;
#pragma unroll
        for (int u = 7; u >= 0; --u) {
            sl[u][0] = r0;
            sl[u][1] = r1;
            r0 *= a0[u];
            r1 *= a1[u];
        }
        *reinterpret_cast<float2 *>(htot + gh * 64 + 2 * lane) = make_float2(pl[7][0], pl[7][1]);
        const float qm = fmaxf(__low2float(qm2), __high2float(qm2));
        const float km = fmaxf(__low2float(km2), __high2float(km2));
        const unsigned wq = __reduce_max_sync(0xffffffffu, __float_as_uint(qm));
        const unsigned wk = __reduce_max_sync(0xffffffffu, __float_as_uint(km));
        if (lane == 0) {
            atomicMax(&qmax[gI], wq);
            atomicMax(kmax, wk);
        }
    }
    named_sync(kBarA, kThreadsA);
    // ---------- chunk factors for my two channels
    float dch[2], bef[2], aft[2];
    bool bad = __uint_as_float(*kmax) > kFastMaxK;
    {
        float2 ht[8];
#pragma unroll
        for (int h8 = 0; h8 < 8; ++h8) ht[h8] = *reinterpret_cast<const float2 *>(htot + h8 * 64 + 2 * lane);
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            float d = 1.f, bf = 1.f, af = 1.f;
#pragma unroll
            for (int h8 = 0; h8 < 8; ++h8) {
                const float x = e ? ht[h8].y : ht[h8].x;
                d *= x;
                if (h8 < gh) bf *= x;
                if (h8 > gh) af *= x;
            }
            dch[e] = d;
            bef[e] = bf;
            aft[e] = af;
            bad |= !(d >= kFastMinDecay);
        }
    }
    // every warp's lanes cover all 64 channels and kmax is already reduced, so a warp
    // vote gives each warp the chunk's decision without a group barrier
    const bool slow = __any_sync(0xffffffffu, bad);
    const float2 dc = *reinterpret_cast<const float2 *>(dcum + (held ? ci : 0) * 64 + 2 * lane);
    if (gh == 0) {
        *reinterpret_cast<float2 *>(sm + L::dloc + b * 256 + 8 * lane) = make_float2(dch[0], dch[1]);
        if (ci + 1 <= kMaxSpan) {
            const float2 d0 = *reinterpret_cast<const float2 *>(dcum + ci * 64 + 2 * lane);
            *reinterpret_cast<float2 *>(dcum + (ci + 1) * 64 + 2 * lane) =
                make_float2(d0.x * dch[0], d0.y * dch[1]);
        }
    }
    if (!slow) {
        // ---------- fast path: Qint = q P, K~ = k / P (= k * suffix / d)
        // The factors (P in [e^-6, 1], suffix / d in [1, e^6]) are rounded to fp16 and
        // applied with packed fp16 multiplies (d >= e^-6 here: the fast division's
        // couple of ulp vanish in that rounding).
        const float i0 = __fdividef(aft[0], dch[0]), i1 = __fdividef(aft[1], dch[1]);
        const __half2 dch2 = __floats2half2_rn(dc.x, dc.y);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const uint32_t o = sw_off(gt0 + u, 2 * lane);
            const __half2 qi = __hmul2(qh[u], __floats2half2_rn(pl[u][0] * bef[0], pl[u][1] * bef[1]));
            *reinterpret_cast<__half2 *>(qo + o) = qi;
            if (held) *reinterpret_cast<__half2 *>(qr + o) = __hmul2(qi, dch2);
            *reinterpret_cast<__half2 *>(ko + o) = __hmul2(kh[u], __floats2half2_rn(sl[u][0] * i0, sl[u][1] * i1));
        }
    } else {
        // ---------- sub-block path: 16-token sub-blocks, factors <= 1 off the diagonal
        float T[4][2];
#pragma unroll
        for (int L4 = 0; L4 < 4; ++L4) {
            const float2 h0 = *reinterpret_cast<const float2 *>(htot + (2 * L4) * 64 + 2 * lane);
            const float2 h1 = *reinterpret_cast<const float2 *>(htot + (2 * L4 + 1) * 64 + 2 * lane);
            T[L4][0] = h0.x * h1.x;
            T[L4][1] = h0.y * h1.y;
        }
        bool dbad = false;
#pragma unroll
        for (int L4 = 0; L4 < 4; ++L4)
            if (L4 == gI) dbad |= !(T[L4][0] >= kDiagMinTotal) || !(T[L4][1] >= kDiagMinTotal);
        dbad |= __uint_as_float(qmax[gI]) > kDiagMaxQ;
        if (__any_sync(0xffffffffu, dbad) && lane == 0) atomicOr(&flags[gI], 1);
        named_sync(kBarA, kThreadsA);
        const int anyflag = flags[0] | flags[1] | flags[2] | flags[3];
        if (anyflag) {
            for (int pr = tid; pr < 4 * 256; pr += kThreadsA) {
                const int I = pr >> 8, u = (pr >> 4) & 15, w = pr & 15;
                if (!flags[I] || w > u) continue;
                const int tu = I * kSub + u, tw = I * kSub + w;
                float acc = 0.f;
                if (tu < nrows) {
                    for (int i = 0; i < kDK; ++i) {
                        float lg = 0.f;
                        for (int r2 = tw + 1; r2 <= tu; ++r2)
                            lg += gate1<kZ>(__half2float(*reinterpret_cast<const __half *>(st + 2 * kTile + r2 * 128 + 2 * i)), inv_tau);
                        const float qv = __half2float(*reinterpret_cast<const __half *>(st + tu * 128 + 2 * i));
                        const float kv = __half2float(*reinterpret_cast<const __half *>(st + kTile + tw * 128 + 2 * i));
                        acc += qv * kv * exp_f(lg);
                    }
                }
                diagx[(I * 16 + u) * 16 + w] = acc;
            }
        }
        // MMA 1 of the previous chunk may still read qj / kbar
        if (ci > 0) {
            wait_phase(bar(sm, B_MMA1 + (b ^ 1)), m1_seen, m1_prev, to);
            tc_fence_after();
        }
        named_sync(kBarA, kThreadsA);
        const bool diag_bad = flags[gI] != 0;
        float cf[2][4], bI[2], aI[2], hin[2], hout[2];
        const float2 h0 = *reinterpret_cast<const float2 *>(htot + (2 * gI) * 64 + 2 * lane);
        const float2 h1 = *reinterpret_cast<const float2 *>(htot + (2 * gI + 1) * 64 + 2 * lane);
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            float b0 = 1.f, a0 = 1.f, tI = 1.f;
#pragma unroll
            for (int L4 = 0; L4 < 4; ++L4) {
                if (L4 < gI) b0 *= T[L4][e];
                if (L4 > gI) a0 *= T[L4][e];
                if (L4 == gI) tI = T[L4][e];
            }
            bI[e] = b0;
            aI[e] = a0;
#pragma unroll
            for (int J = 0; J < 4; ++J) {
                float cj = 1.f;
#pragma unroll
                for (int L4 = 0; L4 < 4; ++L4)
                    if (L4 > J && L4 < gI) cj *= T[L4][e];
                cf[e][J] = (J == gI) ? (diag_bad ? 0.f : 1.f / tI) : cj;
            }
            hin[e] = ghf ? (e ? h0.y : h0.x) : 1.f;
            hout[e] = ghf ? 1.f : (e ? h1.y : h1.x);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int t = gt0 + u;
            const uint32_t o = sw_off(t, 2 * lane);
            const float2 qv = __half22float2(qh[u]);
            const float2 kv = __half22float2(kh[u]);
            const float qp0 = qv.x * (pl[u][0] * hin[0]);
            const float qp1 = qv.y * (pl[u][1] * hin[1]);
            const float ks0 = kv.x * (sl[u][0] * hout[0]);
            const float ks1 = kv.y * (sl[u][1] * hout[1]);
            st_h2(qo + o, qp0 * bI[0], qp1 * bI[1]);
            if (held) st_h2(qr + o, qp0 * bI[0] * dc.x, qp1 * bI[1] * dc.y);
            st_h2(sm + L::kbar + o, ks0, ks1);
            st_h2(ko + o, ks0 * aI[0], ks1 * aI[1]);
#pragma unroll
            for (int J = 0; J < 4; ++J)
                if (J <= gI)
                    st_h2(sm + L::qj + L::qj_region(J) + sw_off(t - 16 * J, 2 * lane), qp0 * cf[0][J],
                          qp1 * cf[1][J]);
        }
    }
    fence_proxy_async_cta();
    named_sync(kBarA, kThreadsA);
    if (tid == 0) {
        mbar_arrive(bar(sm, B_STGE + b));   // the loader may refill this staging buffer
        *misc_slow(sm, b) = slow ? 1 : 0;
        mbar_arrive(bar(sm, B_GATE + b));   // operands ready: MMA 1 may be issued
    }
    if (tid == 64) {   // max |q| of the chunk (for the phase-4 bound); clear the maxima
        const unsigned m = max(max(qmax[0], qmax[1]), max(qmax[2], qmax[3]));
        if (ci < kMaxSpan) reinterpret_cast<float *>(sm + L::cmeta)[2 * ci] = __uint_as_float(m);
        qmax[0] = qmax[1] = qmax[2] = qmax[3] = 0u;
        *kmax = 0u;
    }
    return slow;
}

// MMA 1 of the chunk in buffer b (one thread): dS = K~^T V into TMEM dS buffer b,
// scores = Qint K~^T (or the four sub-block products) into the scores columns.
// (Called by a whole converged warp; one elected lane issues.)
__device__ __forceinline__ void issue_mma1(uint32_t sbase, uint32_t tmem, int b, int vb, bool slow,
                                           uint64_t *done) {
    tc_fence_after();
    const uint32_t kta = sbase + L::kt + b * kTile;
    const uint32_t va = sbase + L::vop + vb * kTile;
    const uint32_t qa = sbase + L::qint + b * kTile;
    if (!slow) {
        uint64_t d_k[4], d_v[4], d_q[4], d_kr[4];
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            d_k[kk] = desc_sw128(kta + kk * 2048, kTile, 1024);
            d_v[kk] = desc_sw128(va + kk * 2048, kTile, 1024);
            d_q[kk] = desc_sw128(qa + kk * 32, 16, 1024);
            d_kr[kk] = desc_sw128(kta + kk * 32, 16, 1024);
        }
        if (elect_one_sync()) {
            constexpr uint32_t id_ds = idesc_f16_f32(64, kDV, true, true);
            constexpr uint32_t id = idesc_f16_f32(64, 64, false, false);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                umma_f16(tmem + kColDS + 64 * b, d_k[kk], d_v[kk], id_ds, kk > 0 ? 1u : 0u);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                umma_f16(tmem + kColScores, d_q[kk], d_kr[kk], id, kk > 0 ? 1u : 0u);
            umma_commit(done);
        }
        __syncwarp();
        return;
    }
    if (elect_one_sync()) {
        constexpr uint32_t id_ds = idesc_f16_f32(64, kDV, true, true);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            umma_f16(tmem + kColDS + 64 * b, desc_sw128(kta + kk * 2048, kTile, 1024),
                     desc_sw128(va + kk * 2048, kTile, 1024), id_ds, kk > 0 ? 1u : 0u);
        constexpr uint32_t id = idesc_f16_f32(64, 16, false, false);
        for (int J = 0; J < 4; ++J) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint32_t aa = sbase + L::qj + L::qj_region(J) - 16 * J * 128 + kk * 32;
                const uint32_t bb = sbase + L::kbar + 16 * J * 128 + kk * 32;
                umma_f16(tmem + kColScores + 16 * J, desc_sw128(aa, 16, 1024),
                         desc_sw128(bb, 16, 1024), id, kk > 0 ? 1u : 0u);
            }
        }
        umma_commit(done);
    }
    __syncwarp();
}

// Group B (warps 8-11), MMA 1 of a chunk complete: TMEM -> registers of the scores
// (columns 64..127).  Warp q holds TMEM lanes 32q.. =
// rows 16q .. 16q+15; thread rows 16q + lane/4 (+8), columns 2 (lane % 4) + 8 j (+1),
// the second register set for columns 32 and up.
struct BRegs {
    uint32_t s0[16], s1[16];
};

__device__ __forceinline__ void load_tmem_b(uint32_t tmem, BRegs &r) {
    const uint32_t ta = tmem + ((uint32_t)(32 * ((threadIdx.x >> 5) & 3)) << 16);
    tc_fence_after();
    tmem_ld_16x256b_x4(ta + kColScores, r.s0);
    tmem_ld_16x256b_x4(ta + kColScores + 32, r.s1);
    tmem_ld_wait();
}

// Causal fp16 P of warp q's rows (16q ..) from its scores registers: column block
// 2 half + cc / 2 (16 columns) lies left of the diagonal for blocks < Q (kept as is),
// right of it for blocks > Q (zero: nothing to convert), and on it for block Q, the
// only one compared element by element (row and column within the block: lane / 4 +
// 8 hh and 2 (lane % 4) + 8 (cc % 2)); with `fb` that block comes from the exact
// diagonal diagx.  v: packed column 4 j + lane % 4 per register, as the TMEM store
// wants it; pmx: max |P|.
template <int Q>
__device__ __forceinline__ void causal_p(const BRegs &r, const float *diagx, bool fb, int lane,
                                         uint32_t (&v)[16], float &pmx) {
    const int rl = lane >> 2, cl = 2 * (lane & 3);
#pragma unroll
    for (int half = 0; half < 2; ++half)
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int blk = 2 * half + (cc >> 1);
                uint32_t &out = v[2 * (cc + 4 * half) + hh];
                if (blk > Q) {
                    out = 0u;
                    continue;
                }
                const uint32_t *rr = half ? r.s1 : r.s0;
                float x0 = __uint_as_float(rr[4 * cc + 2 * hh]);
                float x1 = __uint_as_float(rr[4 * cc + 2 * hh + 1]);
                if (blk == Q) {
                    const int row = rl + 8 * hh, col = cl + 8 * (cc & 1);
                    if (fb) {
                        x0 = diagx[(Q * 16 + row) * 16 + col];
                        x1 = diagx[(Q * 16 + row) * 16 + col + 1];
                    }
                    x0 = col <= row ? x0 : 0.f;
                    x1 = col + 1 <= row ? x1 : 0.f;
                }
                pmx = fmaxf(pmx, fmaxf(fabsf(x0), fabsf(x1)));
                out = pack_half2(x0, x1);
            }
}

// Scores -> causal fp16 P, written back over the scores' own TMEM columns as the A
// operand of MMA 2 (M=64 lane layout, fp16 pairs packed per 32-bit column: the
// thread's pair (row, columns 2k, 2k+1) is packed column k).  With `fb` (this warp's
// sub-block uses the exact diagonal) the diagonal block comes from diag[b].
__device__ __forceinline__ void store_p_tmem(uint8_t *sm, uint32_t tmem, const BRegs &r, int b,
                                             bool fb) {
    const int lane = threadIdx.x & 31, q = (threadIdx.x >> 5) & 3;
    const float *diagx = reinterpret_cast<const float *>(sm + L::diag) + b * 1024;
    uint32_t v[16];
    float pmx = 0.f;
    switch (q) {   // warp-uniform
    case 0: causal_p<0>(r, diagx, fb, lane, v, pmx); break;
    case 1: causal_p<1>(r, diagx, fb, lane, v, pmx); break;
    case 2: causal_p<2>(r, diagx, fb, lane, v, pmx); break;
    default: causal_p<3>(r, diagx, fb, lane, v, pmx); break;
    }
    range_check(pmx);
    asm volatile(
        "tcgen05.st.sync.aligned.16x128b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            tmem + ((uint32_t)(32 * q) << 16) + kColScores),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Group A (warps 0-7), MMA 1 of chunk cr complete: TMEM readout of dS(cr) and the
// state update S <- d * S + dS (dS comes scaled by 1/d on the fast path) in the fp32
// tile, d from dloc[b]; the new state also goes to `so_next` (fp16 S_prev operand of
// chunk cr+1's MMA 2) and to `agg` (the span's published aggregate) when non-null.
// Warp w reads TMEM lanes of quarter w % 4 (rows 16 (w % 4) ..) and columns
// 32 (w / 4) ..: 16 elements per thread.  Ends with group A past its writes.
// kLoadFirst: every load of the state tile before any store, so that the loads
// overlap (faster where registers allow: the short-span instance).
template <bool kLoadFirst>
__device__ __forceinline__ void update_state_a(uint8_t *sm, uint32_t tmem, int b, bool slow,
                                               uint8_t *so_next, float *agg) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int sp = warp & 3, chalf = warp >> 2;
    const int rrow0 = 16 * sp + (lane >> 2);
    const int rcol0 = 32 * chalf + 2 * (lane & 3);
    tc_fence_after();
    uint32_t rd[16];
    tmem_ld_16x256b_x4(tmem + ((uint32_t)(32 * sp) << 16) + kColDS + 64 * b + 32 * chalf, rd);
    tmem_ld_wait();
    const float *dloc = reinterpret_cast<const float *>(sm + L::dloc + b * 256);
    uint8_t *sst = sm + L::sst;
    float2 sv[2][4];
    float smx = 0.f;
    if constexpr (kLoadFirst) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                const int i = rrow0 + 8 * hh, col = rcol0 + 8 * cc;
                sv[hh][cc] = *reinterpret_cast<const float2 *>(sst + agg_off(i, col >> 2) + (col & 3) * 4);
            }
    }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        const int i = rrow0 + 8 * hh;
        const float di = dloc[i];
        const float scl = slow ? 1.f : di;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
            const int col = rcol0 + 8 * cc;
            float2 *sp2 = reinterpret_cast<float2 *>(sst + agg_off(i, col >> 2) + (col & 3) * 4);
            const float2 s = kLoadFirst ? sv[hh][cc] : *sp2;
            const float2 sn = make_float2(fmaf(di, s.x, scl * __uint_as_float(rd[4 * cc + 2 * hh])),
                                          fmaf(di, s.y, scl * __uint_as_float(rd[4 * cc + 2 * hh + 1])));
            *sp2 = sn;
            smx = fmaxf(smx, fmaxf(fabsf(sn.x), fabsf(sn.y)));
            if (so_next != nullptr) st_h2(so_next + sw_off(i, col), sn.x, sn.y);
            if (agg != nullptr) *reinterpret_cast<float2 *>(agg + i * kDV + col) = sn;
        }
    }
    if (so_next != nullptr) range_check(smx);   // the fp16 S_prev operand
    tc_fence_before();
    fence_proxy_async_cta();
    named_sync(kBarA, kThreadsA);
}

// Loader warp: chunk c of the span into staging buffer c % 2 and V tile c % 3 once
// group A is done with the staging buffer (chunk c-2) and MMA 2 with the V tile
// (chunk c-3).
template <int NL>
__device__ __forceinline__ void loader_load(const Params &P, uint8_t *sm, int seq, int c0, int c,
                                            int lane, int lw, uint32_t (&nuse)[2], uint32_t (&nvuse)[3],
                                            bool &to) {
    const int b = c & 1, vb = c % 3;
    wait_l(bar(sm, B_STGE + b), (nuse[b] & 1u) ^ 1u, to);
    wait_l(bar(sm, B_VE + vb), (nvuse[vb] & 1u) ^ 1u, to);
    ++nuse[b];
    ++nvuse[vb];
    load_chunk<NL>(P, sm, seq, c0 + c, b, vb, lane, lw);
    cp_async_mbar_arrive_noinc(bar(sm, B_STGF + b));
}

// Phase 4 (all threads): cp.async of chunk c's q, g rows and stored output rows into
// three unswizzled tiles (row t at byte t * 128) at dst_q, dst_g, dst_o; one group.
// (Out of line, scalar arguments: it runs once per span and adds nothing to the
// register pressure of the kernel body.)
__device__ __noinline__ void load_qgo(const __half *q, const __half *g, const __half *o, int N, int H,
                                      int W, int dir, int heads, int seq, int c, uint32_t dst_q,
                                      uint32_t dst_g, uint32_t dst_o, int nthreads, int ldk, int ldv) {
    const int bq = seq / heads, hq = seq - bq * heads;
    const int p0 = c * kChunk;
    for (int x = (int)threadIdx.x; x < 3 * 64 * 8; x += nthreads) {
        const int ten = x / 512, rem = x - ten * 512, t = rem >> 3, pc = rem & 7;
        const bool ok = p0 + t < N;
        size_t ro = 0;
        if (ok) ro = (size_t)((bq * N + scan_to_token(p0 + t, H, W, dir)) * heads + hq);
        const __half *src = ten == 0 ? q + ro * ldk : (ten == 1 ? g + ro * ldk : o + ro * ldv);
        const uint32_t d = ten == 0 ? dst_q : (ten == 1 ? dst_g : dst_o);
        cp_async16(d + t * 128 + 16 * pc, src + 8 * pc, ok ? 16u : 0u);
    }
    cp_async_commit();
}

// Phase 4 (all threads; groups A's 256 threads compute): Qint * D_c of a chunk from
// its raw q, g rows (qs, gs: unswizzled) and the decay product D_c from the span start
// (dc), into the swizzled K-major tile dst.  Thread layout as in gating.  (Out of
// line: once per span.)
template <bool kZ>
__device__ __noinline__ void rebuild_qd(uint8_t *sm, const uint8_t *qs, const uint8_t *gs,
                                        const float *dc, uint8_t *dst, float inv_tau) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    float *htot = reinterpret_cast<float *>(sm + L::htot);
    const int gI = warp >> 1, ghf = warp & 1, gt0 = 16 * gI + 8 * ghf, gh = 2 * gI + ghf;
    float pl[8][2];
    if (warp < 8) {
        float r0 = 1.f, r1 = 1.f;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const float2 gv = gate2<kZ>(ld_h2(gs + (gt0 + u) * 128 + 4 * lane), inv_tau);
            r0 *= exp_f(gv.x);
            r1 *= exp_f(gv.y);
            pl[u][0] = r0; pl[u][1] = r1;
        }
        *reinterpret_cast<float2 *>(htot + gh * 64 + 2 * lane) = make_float2(r0, r1);
    }
    __syncthreads();
    if (warp < 8) {
        float bf0 = 1.f, bf1 = 1.f;
        for (int h8 = 0; h8 < gh; ++h8) {
            const float2 x = *reinterpret_cast<const float2 *>(htot + h8 * 64 + 2 * lane);
            bf0 *= x.x;
            bf1 *= x.y;
        }
        const float D0 = dc[2 * lane] * bf0, D1 = dc[2 * lane + 1] * bf1;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const float2 qv = ld_h2(qs + (gt0 + u) * 128 + 4 * lane);
            st_h2(dst + sw_off(gt0 + u, 2 * lane), qv.x * pl[u][0] * D0, qv.y * pl[u][1] * D1);
        }
    }
}

// Group B (warps 8-11): the state update S <- d * S + dS of a chunk (as group A's,
// with 32 elements per thread: warp bw reads TMEM lanes of quarter bw, all 64 columns)
// into the fp32 tile and to `agg`.  Used by the short-span instance for the span's last
// chunk, which group B reaches first (its held chunks need no epilogue in phase 1).
// `agg` is written in fragment order, so that every warp store is 512 contiguous
// bytes: float4 number 256 k + s holds, for slot s = 32 w + l (w < 8: quarter w % 4,
// column half w / 4; l a lane), row 16 (w % 4) + l / 4 + 8 (k / 2) and columns
// c, c + 1, c + 8, c + 9 with c = 32 (w / 4) + 2 (l % 4) + 16 (k % 2).
__device__ __forceinline__ void update_state_b(uint8_t *sm, uint32_t tmem, int b, bool slow, float *agg,
                                               int bw, int lane) {
    const int row0 = 16 * bw + (lane >> 2), col0 = 2 * (lane & 3);
    uint32_t r0[16], r1[16];
    const uint32_t ta = tmem + ((uint32_t)(32 * bw) << 16) + kColDS + 64 * b;
    tmem_ld_16x256b_x4(ta, r0);
    tmem_ld_16x256b_x4(ta + 32, r1);
    tmem_ld_wait();
    const float *dloc = reinterpret_cast<const float *>(sm + L::dloc + b * 256);
    uint8_t *sst = sm + L::sst;
    // every load of the state before any store, so that the loads overlap
    float2 sq[2][2][4];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int x = 0; x < 2; ++x)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int i = row0 + 8 * h, col = col0 + 8 * j + 32 * x;
                sq[h][x][j] = *reinterpret_cast<const float2 *>(sst + agg_off(i, col >> 2) + (col & 3) * 4);
            }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int i = row0 + 8 * h;
        const float di = dloc[i];
        const float scl = slow ? 1.f : di;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            const uint32_t *rr = x ? r1 : r0;
            float2 sn[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int col = col0 + 8 * j + 32 * x;
                const float2 sv = sq[h][x][j];
                sn[j] = make_float2(fmaf(di, sv.x, scl * __uint_as_float(rr[4 * j + 2 * h])),
                                    fmaf(di, sv.y, scl * __uint_as_float(rr[4 * j + 2 * h + 1])));
                *reinterpret_cast<float2 *>(sst + agg_off(i, col >> 2) + (col & 3) * 4) = sn[j];
            }
            if (agg != nullptr) {
                float4 *a4 = reinterpret_cast<float4 *>(agg) + 32 * (bw + 4 * x) + lane;
                a4[2 * h * 256] = make_float4(sn[0].x, sn[0].y, sn[1].x, sn[1].y);
                a4[(2 * h + 1) * 256] = make_float4(sn[2].x, sn[2].y, sn[3].x, sn[3].y);
            }
        }
    }
}

// L2 prefetch of row x (of 128) of the first two chunks of the span that CTA `blk`
// runs first: its q, k, g and v rows.  It is issued before the wait on the grid
// ahead on the stream: a prefetch moves nothing into the SM and L2 is where every
// SM's accesses meet, so a later write by that grid still reaches this grid's loads.
__device__ __forceinline__ void prefetch_span_rows(const Params &P, const Work &Wk, int blk, int x) {
    const int PS = Wk.P, kspan = blk % PS, seq = blk / PS;
    if (seq >= P.n_seq) return;
    const int c0 = kspan * Wk.Lc;
    if (x >= min(min(Wk.Lc, P.n_chunks - c0), 2) * kChunk) return;
    const int p = c0 * kChunk + x;
    if (p >= P.N) return;
    const int bb = seq / P.heads, hh = seq - bb * P.heads;
    const size_t ro = ((size_t)bb * P.N + scan_to_token(p, P.H, P.W, P.dir)) * P.heads + hh;
    prefetch_l2(P.q + ro * P.ldk);
    prefetch_l2(P.k + ro * P.ldk);
    prefetch_l2(P.g + ro * P.ldk);
    prefetch_l2(P.v + ro * P.ldv);
}

// The span's aggregate state from the fp32 state tile in shared memory to the
// workspace (row-major), nthr threads with consecutive indices from 0: whole float4
// per thread, consecutive threads on consecutive 16 bytes.  (Group A's publish: a
// second pass over the tile measured faster than its update's scattered 8-byte
// stores; group B's four warps store straight from the update.)
__device__ __forceinline__ void store_aggregate(const uint8_t *sm, float *agg, int t, int nthr) {
    const uint8_t *sst = sm + L::sst;
    for (int e = t; e < kDK * kDV / 4; e += nthr)
        reinterpret_cast<float4 *>(agg)[e] = *reinterpret_cast<const float4 *>(sst + agg_off(e >> 4, e & 15));
}

template <int NL, bool kZ>
__global__ void __launch_bounds__(span_threads<NL>(), 1) gla_fwd_span_kernel(const Params P, const Work Wk) {
    constexpr int kThreads = span_threads<NL>();
    extern __shared__ uint8_t smem_raw[];
    // aligned by an offset from the shared array itself (not through an integer), so
    // that the compiler still sees every tile access as shared memory
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int PS = Wk.P;
    const int kspan = (int)blockIdx.x % PS;
    const int grp = (int)blockIdx.x / PS, ngrp = (int)gridDim.x / PS;

    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar(sm, B_TMEM));
    float *dcum = reinterpret_cast<float *>(sm + L::dcum);
    float *cmeta = reinterpret_cast<float *>(sm + L::cmeta);
    int *rowb = reinterpret_cast<int *>(sm + L::rowb);

    // first data into L2 while the grid ahead finishes: this CTA's span and, for long
    // spans, the span of the CTA dispatched last (likely the last to find a free SM;
    // for short spans the extra traffic measured slower)
    if (tid >= 128 && (NL == 2 ? tid < 384 : tid < 256))
        prefetch_span_rows(P, Wk, NL == 2 && tid >= 256 ? (int)(gridDim.x - 1 - blockIdx.x) : (int)blockIdx.x, tid & 127);
    if (warp == 0) {
        tmem_alloc(tmem_slot, kSpanTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(sm, B_STGF + i), 32 * NL);
            mbar_init(bar(sm, B_STGE + i), 1);
            mbar_init(bar(sm, B_OPSE + i), 1);
        }
        for (int i = 0; i < 2; ++i) mbar_init(bar(sm, B_MMA1 + i), 1);
        mbar_init(bar(sm, B_MMA2), 1);
        mbar_init(bar(sm, B_FIX), 1);
        for (int i = 0; i < 2; ++i) mbar_init(bar(sm, B_GATE + i), 1);
        for (int i = 0; i < 2; ++i) mbar_init(bar(sm, B_OPSF + i), 1);
        for (int i = 0; i < 3; ++i) mbar_init(bar(sm, B_VE + i), 1);
        fence_mbar_init();
    }
    if (tid < 32) reinterpret_cast<unsigned *>(sm + L::misc)[tid] = 0u;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // a launch that follows this one on the stream may be scheduled now (it waits
    // below for this grid to complete); this grid waits for the one before it
    // before any global memory access
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    bool to = false;
    // Barrier phase counters.  Each role counts only the barriers it waits on, and
    // every role walks every chunk, so the counts stay consistent across sequences.
    uint32_t nuse[2] = {0u, 0u};        // uses of buffer 0 / 1 (per role)
    uint32_t nvuse[3] = {0u, 0u, 0u};   // loader: uses of V tile 0 / 1 / 2
    uint32_t m1s[2] = {0u, 0u};         // MMA 1 phases observed, per parity
    uint32_t m2_seen = 0, g_seen = 0, n_fix = 0;

    for (int seq = grp; seq < P.n_seq; seq += ngrp) {
        const int c0 = kspan * Wk.Lc;
        const int nch = min(Wk.Lc, P.n_chunks - c0);   // >= 1 (host guarantees)
        const int hold = kspan > 0 ? min(kHold, nch) : 0;
        const bool later = kspan > 0;
        float *agg = (PS > 1 && kspan < PS - 1) ? Wk.ws + ((size_t)seq * PS + kspan) * kAggFloats
                                                : nullptr;
        // ---------------- phase 1 prologue: running state and decay products
        // (groups A and B; the loader warp starts loading the sequence meanwhile)
        if (warp < 12) {
            uint8_t *sst = sm + L::sst;
            for (int e = tid; e < kDK * kDV / 4; e += kThreadsA + kThreadsB) {
                const int i = e >> 4, c4 = e & 15;
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (!later && P.s0 != nullptr)
                    v = *reinterpret_cast<const float4 *>(P.s0 + (size_t)seq * P.sstride + (size_t)i * P.ldv + 4 * c4);
                *reinterpret_cast<float4 *>(sst + agg_off(i, c4)) = v;
                // S_prev of chunk 0, the fp16 operand of its MMA 2
                *reinterpret_cast<uint2 *>(sm + L::sop + sw_off(i, 4 * c4)) =
                    make_uint2(pack_half2(v.x, v.y), pack_half2(v.z, v.w));
                range_check(absmax4(v));
            }
            if (tid < 64) dcum[tid] = 1.f;
            if (tid < kMaxSpan * 2) cmeta[tid] = 0.f;
            fence_proxy_async_cta();
            named_sync(kBarPro, kThreadsA + kThreadsB);
            if (tid == 0) mbar_arrive(bar(sm, B_OPSF));   // S_prev of chunk 0 is ready
        }
        // phase indices at the start of the sequence: chunk c is use c/2 of parity c%2
        const uint32_t m1b0 = m1s[0], m1b1 = m1s[1];

        if (warp < 8) {
            // ================================================= group A
            // Iteration it: gating of chunk it (while MMA 1 of chunk it-1 runs; the
            // loader warp issues MMA 1(it) once it is signalled), then the state update
            // from dS(it-1), i.e. S_prev of chunk it.
            bool slow_prev = false;
            for (int it = 0; it <= nch; ++it) {
                const int b = it & 1;
                bool slow = false;
                if (it < nch) {
                    wait_l(bar(sm, B_STGF + b), nuse[b] & 1u, to);
                    wait_l(bar(sm, B_OPSE + b), (nuse[b] & 1u) ^ 1u, to);
                    ++nuse[b];
                    const int nrows = min(kChunk, P.N - (c0 + it) * kChunk);
                    slow = gate_chunk<kZ>(P, sm, it, b, nrows, it < hold, m1s[b ^ 1],
                                          (b ? m1b0 : m1b1) + ((it - 1) >> 1), to, Wk.inv_tau);
                }
                if (it > 0) {
                    wait_phase(bar(sm, B_MMA1 + (b ^ 1)), m1s[b ^ 1], (b ? m1b0 : m1b1) + ((it - 1) >> 1), to);
                    if constexpr (NL == 4)
                        if (it == nch) break;   // the last update is group B's
                    const bool pub = agg != nullptr && it == nch;
                    update_state_a<NL == 4>(sm, tmem, b ^ 1, slow_prev, it < nch ? sm + L::sop + b * kTile : nullptr,
                                   nullptr);
                    if (pub) {
                        store_aggregate(sm, agg, tid, kThreadsA);
                        // aggregate = (state reached from zero, product of the span's decays)
                        // (the CTA barrier orders every thread's stores before thread 0's
                        // release at gpu scope)
                        if (tid < 64) agg[kDK * kDV + tid] = dcum[nch * 64 + tid];
                        named_sync(kBarA, kThreadsA);
                        if (tid == 0)   // readers to come: spans kspan+1 .. PS-1
                            st_release_gpu(Wk.flags + ((size_t)seq * PS + kspan) * kFlagStride, (unsigned)(PS - 1 - kspan));
                    }
                    if (tid == 0 && it < nch) mbar_arrive(bar(sm, B_OPSF + b));   // S_prev of chunk it
                }
                slow_prev = slow;
            }
        } else if (warp < 12) {
            // ================================================= group B
            const int tb = tid - kThreadsA, bw = warp - 8;
            int *rows2 = rowb + 2 * 64;
            for (int c = 0; c < nch; ++c) {
                const int b = c & 1;
                // (spans of at most kShortSpan chunks hold every chunk's output in TMEM,
                // span 0's too: its epilogues wait until it has published)
                const bool held = NL == 4 || c < hold;
                fill_rows(P, seq, c0 + c, rows2, tb);
                wait_l(bar(sm, B_GATE + b), (g_seen >> b) & 1u, to);   // bit b: parity of GATE[b]
                g_seen ^= 1u << b;
                // MMA 1(c) (one elected lane of warp 8): the scores' TMEM columns are
                // free (MMA 2(c-1), complete, consumed P) and so is the dS buffer (group A
                // read dS(c-2) before gating chunk c)
                if (bw == 0) {
                    __syncwarp();
                    fence_proxy_async_cta();
                    issue_mma1(sbase, tmem, b, c % 3, *misc_slow(sm, b) != 0, bar(sm, B_MMA1 + b));
                }
                wait_phase(bar(sm, B_MMA1 + b), m1s[b], (b ? m1b1 : m1b0) + (c >> 1), to);
                BRegs r;
                load_tmem_b(tmem, r);
                store_p_tmem(sm, tmem, r, b, misc_flags(sm, b)[warp & 3] != 0);
                tc_fence_before();
                named_sync(kBarB, kThreadsB);
                if (bw == 0) {
                    // only the issuing warp (converged) waits for S_prev of chunk c (a
                    // lagging waiter could miss a phase: the next one follows MMA 2 of
                    // chunk c); one elected lane issues
                    wait_l(bar(sm, B_OPSF + b), nuse[b] & 1u, to);
                    ++nuse[b];
                    __syncwarp();
                    tc_fence_after();
                    const uint32_t dcol = held ? kColHold + 64 * c : kColWork;
                    const uint32_t qa = sbase + L::qint + b * kTile;
                    const uint32_t sa = sbase + L::sop + b * kTile;
                    const uint32_t va = sbase + L::vop + (c % 3) * kTile;
                    uint64_t d_q[4], d_s[4], d_v[4];
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        d_q[kk] = desc_sw128(qa + kk * 32, 16, 1024);
                        d_s[kk] = desc_sw128(sa + kk * 2048, kTile, 1024);
                        d_v[kk] = desc_sw128(va + kk * 2048, kTile, 1024);
                    }
                    if (elect_one_sync()) {
                        constexpr uint32_t id = idesc_f16_f32(64, kDV, false, true);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_f16(tmem + dcol, d_q[kk], d_s[kk], id, kk > 0 ? 1u : 0u);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)   // P from TMEM: K step 16 = 8 packed columns
                            umma_f16_ta(tmem + dcol, tmem + kColScores + 8 * kk, d_v[kk], id, 1u);
                        umma_commit(bar(sm, B_MMA2));
                        umma_commit(bar(sm, B_OPSE + b));    // Qint, S_prev tiles free
                        umma_commit(bar(sm, B_VE + c % 3));  // V tile free
                    }
                    __syncwarp();
                }
                if constexpr (NL == 4) {
                    if (c == nch - 1) {
                        // the span's last update (group A's ended with chunk c-1's, which
                        // warp 8 has seen: S_prev of chunk c), then the publish
                        named_sync(kBarB, kThreadsB);
                        tc_fence_after();
                        const bool slw = *misc_slow(sm, b) != 0;
                        update_state_b(sm, tmem, b, slw, agg, bw, lane);
                        if (agg != nullptr) {
                            if (tb < 64) agg[kDK * kDV + tb] = dcum[nch * 64 + tb];
                            named_sync(kBarB, kThreadsB);
                            if (tb == 0)   // readers to come: spans kspan+1 .. PS-1
                                st_release_gpu(Wk.flags + ((size_t)seq * PS + kspan) * kFlagStride,
                                               (unsigned)(PS - 1 - kspan));
                        }
                    }
                }
                wait_l(bar(sm, B_MMA2), m2_seen & 1u, to);
                ++m2_seen;
                tc_fence_after();
                if (!held) {
                    // the P tile is free again: it stages the outputs
                    const float mx = store_chunk_out(P, tmem, kColWork, bw, lane, tb, nullptr, kBarB,
                                                     sm + L::p, rows2);
                    if (later && c < kMaxSpan) {
                        const unsigned w = __reduce_max_sync(0xffffffffu, __float_as_uint(mx));
                        if (lane == 0) atomicMax(reinterpret_cast<unsigned *>(cmeta + 2 * c + 1), w);
                    }
                }
            }
        } else {
            // ================================================= loaders (warps 12 ..)
            // Loads run ahead as the staging buffers (once gated) and the V tiles (once
            // MMA 2 has read them) free up.
            for (int c = 0; c < nch; ++c) loader_load<NL>(P, sm, seq, c0, c, lane, warp - 12, nuse, nvuse, to);
        }
        __syncthreads();
        if constexpr (NL == 4) {
            // ---------------- phases 3-5 of a later span of at most kShortSpan chunks
            // Every chunk is held (hold == nch): the S_in term needs only the fp16 S_in
            // tile, and the last span's final state D_span * S_in + S_local is written
            // as S_in is formed, so S_in never goes through shared memory in fp32.
            if (later) {
                // row tables of each epilogue team's first chunk, while the flags come in
                if (warp < 12 && (warp >> 2) < hold)
                    fill_rows(P, seq, c0 + (warp >> 2), rowb + 64 * (warp >> 2), tid - 128 * (warp >> 2));
                // S_in = sum_j (prod_{l>j} D_l) * S_j by Horner over j = 0 .. kspan-1, from
                // the aggregates copied into the phase-1 buffers below the S_in operand
                // tile (kFoldSlots at a time): warp u waits for span j0 + u's flag and copies
                // that aggregate at once (cp.async, no registers held), so the copies
                // overlap the flags' arrival; then each thread forms two float4 of S_in
                // from shared memory (fragment order, as group B's update stores the
                // aggregates: rows i and i + 8, columns c, c + 1, c + 8, c + 9).
                static_assert(kDK * kDV / 4 == 2 * kThreads, "two float4 of S_in per thread");
                constexpr int kAggBytes = kAggFloats * 4;
                constexpr int kFoldSlots = L::sop / kAggBytes;
                static_assert(kFoldSlots >= 1 && kAggBytes % 16 == 0, "fold slots");
                {
                    const float *wseq = Wk.ws + (size_t)seq * PS * kAggFloats;
                    const int e0 = tid, e1 = tid + kThreads;
                    const int sl = tid & 255, fw = sl >> 5, fl = sl & 31;
                    const int i0 = 16 * (fw & 3) + (fl >> 2), i1 = i0 + 8;
                    const int ca = 32 * (fw >> 2) + 2 * (fl & 3) + 16 * (tid >> 8), cb = ca + 8;
                    float4 s0 = make_float4(0.f, 0.f, 0.f, 0.f), s1 = s0;
                    for (int j0 = 0; j0 < kspan; j0 += kFoldSlots) {
                        const int nj = min(kFoldSlots, kspan - j0);
                        for (int u = warp; u < nj; u += kThreads / 32) {
                            unsigned *f = Wk.flags + ((size_t)seq * PS + j0 + u) * kFlagStride;
                            int ok = 1;
                            if (lane == 0) {
                                ok = flag_wait_bounded(f, kWaitLimitNs) ? 1 : 0;
                                if (ok) {
                                    red_dec_gpu(f);   // one reader fewer to come
                                } else {
                                    to = true;
                                    set_error(kErrTimeout);
                                }
                            }
                            // (the warp's copies follow lane 0's acquire)
                            ok = __shfl_sync(0xffffffffu, ok, 0);
                            if (ok) {
                                const float *src = wseq + (size_t)(j0 + u) * kAggFloats;
                                const uint32_t dst = sbase + u * kAggBytes;
                                for (int x = lane; x < kAggBytes / 16; x += 32) cp_async16(dst + 16 * x, src + 4 * x, 16);
                            }
                        }
                        cp_async_commit();
                        cp_async_wait_all();
                        __syncthreads();
                        for (int u = 0; u < nj; ++u) {   // (D_j <= 1: the zero start stays zero)
                            const float *a = reinterpret_cast<const float *>(sm + u * kAggBytes);
                            const float4 a0 = reinterpret_cast<const float4 *>(a)[e0];
                            const float4 a1 = reinterpret_cast<const float4 *>(a)[e1];
                            const float d0 = a[kDK * kDV + i0], d1 = a[kDK * kDV + i1];
                            s0.x = fmaf(d0, s0.x, a0.x);
                            s0.y = fmaf(d0, s0.y, a0.y);
                            s0.z = fmaf(d0, s0.z, a0.z);
                            s0.w = fmaf(d0, s0.w, a0.w);
                            s1.x = fmaf(d1, s1.x, a1.x);
                            s1.y = fmaf(d1, s1.y, a1.y);
                            s1.z = fmaf(d1, s1.z, a1.z);
                            s1.w = fmaf(d1, s1.w, a1.w);
                        }
                        if (j0 + kFoldSlots < kspan) __syncthreads();   // the slots are reused
                    }
                    uint8_t *bt = sm + L::sop;
                    *reinterpret_cast<uint32_t *>(bt + sw_off(i0, ca)) = pack_half2(s0.x, s0.y);
                    *reinterpret_cast<uint32_t *>(bt + sw_off(i0, cb)) = pack_half2(s0.z, s0.w);
                    *reinterpret_cast<uint32_t *>(bt + sw_off(i1, ca)) = pack_half2(s1.x, s1.y);
                    *reinterpret_cast<uint32_t *>(bt + sw_off(i1, cb)) = pack_half2(s1.z, s1.w);
                    range_check(fmaxf(absmax4(s0), absmax4(s1)));   // the fp16 S_in operand
                    if (kspan == PS - 1 && P.sf != nullptr) {
                        // final state of the sequence: D_span * S_in + S_local
                        const uint8_t *sst = sm + L::sst;
                        const auto st2 = [&](int i, int col) {
                            return *reinterpret_cast<const float2 *>(sst + agg_off(i, col >> 2) + (col & 3) * 4);
                        };
                        const float g0 = dcum[nch * 64 + i0], g1 = dcum[nch * 64 + i1];
                        const float2 f0a = st2(i0, ca), f0b = st2(i0, cb), f1a = st2(i1, ca), f1b = st2(i1, cb);
                        float *sf = P.sf + (size_t)seq * P.sstride;
                        *reinterpret_cast<float2 *>(sf + i0 * P.ldv + ca) = make_float2(fmaf(g0, s0.x, f0a.x), fmaf(g0, s0.y, f0a.y));
                        *reinterpret_cast<float2 *>(sf + i0 * P.ldv + cb) = make_float2(fmaf(g0, s0.z, f0b.x), fmaf(g0, s0.w, f0b.y));
                        *reinterpret_cast<float2 *>(sf + i1 * P.ldv + ca) = make_float2(fmaf(g1, s1.x, f1a.x), fmaf(g1, s1.y, f1a.y));
                        *reinterpret_cast<float2 *>(sf + i1 * P.ldv + cb) = make_float2(fmaf(g1, s1.z, f1b.x), fmaf(g1, s1.w, f1b.y));
                    }
                }
                fence_proxy_async_cta();
                __syncthreads();
                // the term for every chunk: one MMA per chunk onto its output in TMEM
                if (warp == 0) {
                    tc_fence_after();
                    if (elect_one_sync()) {
                        constexpr uint32_t id = idesc_f16_f32(64, kDV, false, true);
                        const uint32_t ba = sbase + L::sop;
                        for (int ci = 0; ci < hold; ++ci) {
                            const uint32_t qa = sbase + L::ring + ci * kTile;
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                umma_f16(tmem + kColHold + 64 * ci, desc_sw128(qa + kk * 32, 16, 1024),
                                         desc_sw128(ba + kk * 2048, kTile, 1024), id, 1u);
                        }
                        umma_commit(bar(sm, B_FIX));
                    }
                    __syncwarp();
                }
                wait_l(bar(sm, B_FIX), n_fix & 1u, to);
                ++n_fix;
                tc_fence_after();
                // epilogues: three teams of four warps, chunk ci on team ci % 3
                if (warp < 12) {
                    const int team = warp >> 2, tb = tid - 128 * team, bw = warp & 3;
                    int *rows = rowb + 64 * team;
                    uint8_t *os = sm + L::stg + team * kTile;
                    for (int ci = team; ci < hold; ci += 3) {
                        if (ci != team) {   // (the first chunk's rows are in place)
                            fill_rows(P, seq, c0 + ci, rows, tb);
                            named_sync(3 + team, 128);
                        }
                        store_chunk_out(P, tmem, kColHold + 64 * ci, bw, lane, tb, nullptr, 3 + team, os, rows);
                    }
                }
            } else {
                // span 0: its outputs, complete in TMEM (group B saw every MMA 2 complete)
                tc_fence_after();
                if (warp < 12) {
                    const int team = warp >> 2, tb = tid - 128 * team, bw = warp & 3;
                    int *rows = rowb + 64 * team;
                    uint8_t *os = sm + L::stg + team * kTile;
                    for (int ci = team; ci < nch; ci += 3) {
                        fill_rows(P, seq, c0 + ci, rows, tb);
                        named_sync(3 + team, 128);
                        store_chunk_out(P, tmem, kColHold + 64 * ci, bw, lane, tb, nullptr, 3 + team, os, rows);
                    }
                }
            }
        }
        // ---------------- phase 3: look back over the earlier spans
        // Chunk kHold, the first past the held ones, is the one whose S_in term is
        // usually not negligible: its q, g and stored output rows start loading now
        // into the free V tiles, whether or not it turns out to need them.
        // (Long spans only: the four-loader instance serves spans of at most
        // kShortSpan <= kHold chunks.)
        const bool ext = NL == 2 && later && hold == kHold && nch > kHold;
        if constexpr (NL == 2) if (ext) {
            const uint32_t vo = smem_u32(sm + L::vop);
            load_qgo(P.q, P.g, P.out, P.N, P.H, P.W, P.dir, P.heads, seq, c0 + kHold, vo, vo + kTile,
                     vo + 2 * kTile, kThreads, P.ldk, P.ldv);
        }
        if (NL == 2 && later) {
            if (tid < kspan) {
                unsigned *f = Wk.flags + ((size_t)seq * PS + tid) * kFlagStride;
                if (flag_wait_bounded(f, kWaitLimitNs)) {
                    red_dec_gpu(f);   // one reader fewer to come
                } else {
                    to = true;
                    set_error(kErrTimeout);
                }
            }
            __syncthreads();
            // S_in = S_out(span 0), then S_in = D_j * S_in + S_j for j = 1 .. kspan-1
            float *sin = reinterpret_cast<float *>(sm + L::sin);
            unsigned *rmax = reinterpret_cast<unsigned *>(sm + L::rmax);
            if (tid < 64) rmax[tid] = 0u;
            __syncthreads();
            const float *wseq = Wk.ws + (size_t)seq * PS * kAggFloats;
            for (int e = tid; e < kDK * kDV / 4; e += kThreads) {
                const int i = e >> 4, c4 = e & 15;
                float4 s = __ldcg(reinterpret_cast<const float4 *>(wseq) + e);
                // the later aggregates, four loads in flight at a time
                for (int j0 = 1; j0 < kspan; j0 += 4) {
                    float4 a[4];
                    float dj[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        if (j0 + u < kspan) {
                            const float *wj = wseq + (size_t)(j0 + u) * kAggFloats;
                            a[u] = __ldcg(reinterpret_cast<const float4 *>(wj) + e);
                            dj[u] = __ldcg(wj + kDK * kDV + i);
                        }
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        if (j0 + u < kspan) {
                            s.x = fmaf(dj[u], s.x, a[u].x);
                            s.y = fmaf(dj[u], s.y, a[u].y);
                            s.z = fmaf(dj[u], s.z, a[u].z);
                            s.w = fmaf(dj[u], s.w, a[u].w);
                        }
                    }
                }
                *reinterpret_cast<float4 *>(reinterpret_cast<uint8_t *>(sin) + agg_off(i, c4)) = s;
                const float m = fmaxf(fmaxf(fabsf(s.x), fabsf(s.y)), fmaxf(fabsf(s.z), fabsf(s.w)));
                atomicMax(rmax + i, __float_as_uint(m));   // non-negative: integer order = float order
            }
            __syncthreads();   // S_in and its row maxima complete
            // Chunks past the held ones: is the term negligible?  One warp per chunk:
            //   |term[t][j]| <= max|q| * sum_i D_c[i] * max_j |S_in[i][j]|   (P_t <= 1),
            // negligible when below 2^-16 of the chunk's largest output, i.e. under a
            // 32nd of the fp16 rounding step of that output.  (Later spans have at most
            // kMaxSpan chunks.)
            {
                const float *rmf = reinterpret_cast<const float *>(rmax);
                int *skipf = reinterpret_cast<int *>(sm + L::skipf);
                for (int ci = hold + warp; ci < nch; ci += kThreads / 32) {
                    float part = fmaf(dcum[ci * 64 + 2 * lane], rmf[2 * lane],
                                      dcum[ci * 64 + 2 * lane + 1] * rmf[2 * lane + 1]);
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
                    if (lane == 0) skipf[ci] = cmeta[2 * ci] * part <= 1.52587890625e-5f * cmeta[2 * ci + 1];
                }
            }
            __syncthreads();
        }

        // ---------------- phase 4: add the S_in term to this span's outputs
        if (NL == 2 && later) {
            const float *sin = reinterpret_cast<const float *>(sm + L::sin);
            // held chunks: their ring tiles hold Qint * D_c, so one B tile (S_in, fp16)
            // serves them all; the MMAs accumulate onto the chunks' outputs in TMEM
            if (hold > 0) {
                // chunk kHold, if its term is not negligible, joins them: Qint * D_c rebuilt
                // from the prefetched rows into qint, its correction into the work block,
                // its stored output added in the epilogue
                const bool xfix = ext && !(reinterpret_cast<const int *>(sm + L::skipf))[kHold];
                uint8_t *bt = sm + L::sop;
                for (int e = tid; e < kDK * kDV / 4; e += kThreads) {
                    const int i = e >> 4, c4 = e & 15;
                    const float4 s = *reinterpret_cast<const float4 *>(reinterpret_cast<const uint8_t *>(sin) + agg_off(i, c4));
                    *reinterpret_cast<uint2 *>(bt + sw_off(i, 4 * c4)) =
                        make_uint2(pack_half2(s.x, s.y), pack_half2(s.z, s.w));
                    range_check(absmax4(s));   // the fp16 S_in operand
                }
                if (ext) cp_async_wait_all();   // the prefetch has landed (needed or not)
                __syncthreads();
                if constexpr (NL == 2)
                    if (xfix) rebuild_qd<kZ>(sm, sm + L::vop, sm + L::vop + kTile, dcum + kHold * 64, sm + L::qint, Wk.inv_tau);
                fence_proxy_async_cta();
                __syncthreads();
                if (warp == 0) {
                    tc_fence_after();
                    if (elect_one_sync()) {
                        constexpr uint32_t id = idesc_f16_f32(64, kDV, false, true);
                        const uint32_t ba = smem_u32(bt);
                        for (int ci = 0; ci < hold; ++ci) {
                            const uint32_t qa = sbase + L::ring + ci * kTile;
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                umma_f16(tmem + kColHold + 64 * ci, desc_sw128(qa + kk * 32, 16, 1024),
                                         desc_sw128(ba + kk * 2048, kTile, 1024), id, 1u);
                        }
                        if (xfix) {
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                umma_f16(tmem + kColWork, desc_sw128(sbase + L::qint + kk * 32, 16, 1024),
                                         desc_sw128(ba + kk * 2048, kTile, 1024), id, kk > 0 ? 1u : 0u);
                        }
                        umma_commit(bar(sm, B_FIX));
                    }
                    __syncwarp();
                }
                wait_l(bar(sm, B_FIX), n_fix & 1u, to);
                ++n_fix;
                tc_fence_after();
                // epilogues: three teams of four warps, chunk ci on team ci % 3
                if (warp < 12) {
                    const int team = warp >> 2, tb = tid - 128 * team, bw = warp & 3;
                    int *rows = rowb + 64 * team;
                    uint8_t *os = sm + L::stg + team * kTile;
                    for (int ci = team; ci < hold + (xfix ? 1 : 0); ci += 3) {
                        const bool x = ci == hold;   // chunk kHold: correction + stored output
                        fill_rows(P, seq, c0 + ci, rows, tb);
                        named_sync(3 + team, 128);
                        store_chunk_out(P, tmem, x ? kColWork : kColHold + 64 * ci, bw, lane, tb,
                                        x ? sm + L::vop + 2 * kTile : nullptr, 3 + team, os, rows);
                    }
                }
                __syncthreads();
            }
            // later chunks: exact re-read correction unless the term is provably negligible
            // (spans after the first have at most kMaxSpan chunks)
            const int *skipf = reinterpret_cast<const int *>(sm + L::skipf);
            for (int ci = hold; ci < nch; ++ci) {
                if (skipf[ci] || (ext && ci == kHold)) continue;   // (chunk kHold done above)
                // load q, g, o rows of this chunk (all threads), rebuild Q * P * D_c (long
                // spans: out of line, which measured faster there; short spans keep the
                // inline form, which measured faster for them)
                if constexpr (NL == 2) {
                    const uint32_t stq = smem_u32(sm + L::stg);
                    load_qgo(P.q, P.g, P.out, P.N, P.H, P.W, P.dir, P.heads, seq, c0 + ci, stq,
                             stq + 2 * kTile, stq + 3 * kTile, kThreads, P.ldk, P.ldv);
                    cp_async_wait_all();
                    __syncthreads();
                    rebuild_qd<kZ>(sm, sm + L::stg, sm + L::stg + 2 * kTile, dcum + ci * 64, sm + L::qint, Wk.inv_tau);
                } else {
                    // load q, g, o rows of this chunk (all threads), rebuild Q * P * D_c
                    {
                        const uint32_t stq = smem_u32(sm + L::stg);
                        const int bq = seq / P.heads, hq = seq - bq * P.heads;
                        const int p0 = (c0 + ci) * kChunk;
                        for (int x = tid; x < 3 * 64 * 8; x += kThreads) {
                            const int ten = x / 512, rem = x - ten * 512, t = rem >> 3, pc = rem & 7;
                            const bool ok = p0 + t < P.N;
                            size_t ro = 0;
                            if (ok) ro = (size_t)((bq * P.N + scan_to_token(p0 + t, P.H, P.W, P.dir)) * P.heads + hq);
                            const __half *src = ten == 0 ? P.q + ro * P.ldk : (ten == 1 ? P.g + ro * P.ldk : P.out + ro * P.ldv);
                            const int slot = ten == 0 ? 0 : (ten == 1 ? 2 : 3);
                            cp_async16(stq + slot * kTile + t * 128 + 16 * pc, src + 8 * pc, ok ? 16u : 0u);
                        }
                        cp_async_commit();
                        cp_async_wait_all();
                    }
                    __syncthreads();
                    {
                        // 256 threads: (half-block, channel pair) as in gating; products from the
                        // chunk start
                        float *htot = reinterpret_cast<float *>(sm + L::htot);
                        const int gI = warp >> 1, ghf = warp & 1, gt0 = 16 * gI + 8 * ghf, gh = 2 * gI + ghf;
                        float pl[8][2];
                        if (warp < 8) {
                            float r0 = 1.f, r1 = 1.f;
    #pragma unroll
                            for (int u = 0; u < 8; ++u) {
                                const float2 gv = gate2<kZ>(ld_h2(sm + L::stg + 2 * kTile + (gt0 + u) * 128 + 4 * lane),
                                                            Wk.inv_tau);
                                r0 *= exp_f(gv.x);
                                r1 *= exp_f(gv.y);
                                pl[u][0] = r0; pl[u][1] = r1;
                            }
                            *reinterpret_cast<float2 *>(htot + gh * 64 + 2 * lane) = make_float2(r0, r1);
                        }
                        __syncthreads();
                        if (warp < 8) {
                            float bf0 = 1.f, bf1 = 1.f;
                            for (int h8 = 0; h8 < gh; ++h8) {
                                const float2 x = *reinterpret_cast<const float2 *>(htot + h8 * 64 + 2 * lane);
                                bf0 *= x.x;
                                bf1 *= x.y;
                            }
                            const float D0 = dcum[ci * 64 + 2 * lane] * bf0, D1 = dcum[ci * 64 + 2 * lane + 1] * bf1;
                            uint8_t *qo = sm + L::qint;
    #pragma unroll
                            for (int u = 0; u < 8; ++u) {
                                const float2 qv = ld_h2(sm + L::stg + (gt0 + u) * 128 + 4 * lane);
                                st_h2(qo + sw_off(gt0 + u, 2 * lane), qv.x * pl[u][0] * D0, qv.y * pl[u][1] * D1);
                            }
                        }
                    }
                }
                {
                    // S_in as the fp16 operand
                    uint8_t *bt = sm + L::sop;
                    for (int e = tid; e < kDK * kDV / 4; e += kThreads) {
                        const int i = e >> 4, c4 = e & 15;
                        const float4 s = *reinterpret_cast<const float4 *>(reinterpret_cast<const uint8_t *>(sin) + agg_off(i, c4));
                        *reinterpret_cast<uint2 *>(bt + sw_off(i, 4 * c4)) =
                            make_uint2(pack_half2(s.x, s.y), pack_half2(s.z, s.w));
                        range_check(absmax4(s));   // the fp16 S_in operand
                    }
                }
                fence_proxy_async_cta();
                __syncthreads();
                if (warp == 0) {
                    tc_fence_after();
                    if (elect_one_sync()) {
                        constexpr uint32_t id = idesc_f16_f32(64, kDV, false, true);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_f16(tmem + kColWork, desc_sw128(sbase + L::qint + kk * 32, 16, 1024),
                                     desc_sw128(sbase + L::sop + kk * 2048, kTile, 1024), id, kk > 0 ? 1u : 0u);
                        umma_commit(bar(sm, B_FIX));
                    }
                    __syncwarp();
                }
                wait_l(bar(sm, B_FIX), n_fix & 1u, to);
                ++n_fix;
                tc_fence_after();
                if (warp >= 8 && warp < 12) {
                    const int tb = tid - kThreadsA, bw = warp - 8;
                    fill_rows(P, seq, c0 + ci, rowb + 128, tb);
                    named_sync(kBarB, kThreadsB);
                    store_chunk_out(P, tmem, kColWork, bw, lane, tb, sm + L::stg + 3 * kTile, kBarB,
                                    sm + L::stg + 4 * kTile, rowb + 128);
                }
                __syncthreads();
            }
        }

        // ---------------- phase 5: final state of the sequence
        if (kspan == PS - 1 && P.sf != nullptr && (NL == 2 || !later)) {
            const float *sst = reinterpret_cast<const float *>(sm + L::sst);
            const float *sin = reinterpret_cast<const float *>(sm + L::sin);
            for (int e = tid; e < kDK * kDV / 4; e += kThreads) {
                const int i = e >> 4, c4 = e & 15;
                float4 s = *reinterpret_cast<const float4 *>(reinterpret_cast<const uint8_t *>(sst) + agg_off(i, c4));
                if (later) {
                    const float di = dcum[nch * 64 + i];
                    const float4 a = *reinterpret_cast<const float4 *>(reinterpret_cast<const uint8_t *>(sin) + agg_off(i, c4));
                    s.x = fmaf(di, a.x, s.x);
                    s.y = fmaf(di, a.y, s.y);
                    s.z = fmaf(di, a.z, s.z);
                    s.w = fmaf(di, a.w, s.w);
                }
                *reinterpret_cast<float4 *>(P.sf + (size_t)seq * P.sstride + (size_t)i * P.ldv + 4 * c4) = s;
            }
        }
        __syncthreads();   // staging / state tiles are reused by the next sequence
    }

    // after a timeout some MMA may still be in flight: give it time before freeing TMEM
    if (__syncthreads_or(to)) {
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 1000000ull) {
        }
    }
    if (warp == 0) tmem_dealloc(tmem, kSpanTmemCols);
}

}  // namespace sp
}  // namespace gtr
