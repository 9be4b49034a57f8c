// gla_fwd_pipe.cuh -- TMA-staged, warp-specialised GTR token-mixer forward kernel for
// dk = dv = 64 (included by gtr_gla.cu, which holds the shared helpers and the C ABI).
//
// The forward pass (GTR news article, tokendh.com, section "线性注意力到底在省什么": key-side
// forget gate, value-side decay 1; section "速度到底快在哪，TensorRT部署做了什么": chunkwise,
// FP16 with FP32 accumulation, only the chunk-boundary state passed in order) for one
// (batch, head) sequence, chunk c of 64 scan positions, b = inclusive cumulative sum of the
// log-decay g over the chunk (per key channel), b_C its last row, d = exp(b_C):
//
//     Qint = Q * exp(b)        K~ = K * exp(-b)
//     O    = Qint S_prev + tril(Qint K~^T) V
//     S    = d * (S_prev + K~^T V)
//
// Decomposition.  Each sequence is cut into P spans of chunks; one CTA owns one span
// (persistent CTAs loop over sequences).  Every span runs its chunks from a zero state
// (span 0 from S0), publishes (state reached, product of its decays) to a workspace,
// and the later spans fold their predecessors' aggregates into the true entering state
// S_in and add the missing term (Qint * D_c) S_in to their outputs, D_c being the decay
// product from the span start to chunk c.
//
// Roles (one CTA = 18 warps):
//   warp 0       producer: one lane issues the chunk's TMA tensor copies (q, k, g, v)
//                into a 3-slot staging ring.  The scan direction is applied only in the
//                copies' coordinates: a chunk is a list of runs of grid tokens that are
//                contiguous in memory (a row segment, or a column segment at stride W),
//                each copied in memory order by boxes of 64, 32, .. 1 rows; the lanes
//                write the table staging row <- scan position (identity for L->R and
//                T->B, reversed inside each run for R->L and B->T);
//   warp 1       MMA issuer (one elected lane): MMA 1 = (K~^T V, Qint K~^T) and
//                MMA 2 = Qint S_prev + P V, tcgen05 kind::f16 with fp32 accumulators
//                in tensor memory, P read from tensor memory;
//   warps 2-5    state group U: S (fp32) lives in registers in the accumulator's
//                fragment layout; per chunk S <- d * (S + dS), and its fp16 copy is the
//                next chunk's S_prev operand;
//   warps 6-9    readout group RE: scores -> causal mask -> fp16 P back into tensor
//                memory; then the chunk's output tile -> fp16 -> coalesced row stores;
//   warps 10-17  gating group G: per chunk the cumulative decays, Qint and K~ (or the
//                sub-block operands, below) into 128-byte-swizzled operand tiles, and V
//                into its operand tile in scan order.
// Every hand-off is an mbarrier with a bounded wait; each producer of a double-buffered
// resource waits for its consumer's release of the previous use, so that no waiter can
// fall two phases behind.
//
// Range safety.  The fast path needs every channel's chunk decay d >= e^-6 and |k| <= 100
// (then |K~| <= 403 |k| stays inside fp16).  Otherwise the chunk takes the sub-block path:
// 16-token sub-blocks, the diagonal blocks anchored at their own start and the blocks
// below the diagonal at the end of their key block, so that every factor is a product of
// decays <= 1 except the diagonal keys' (bounded by e^8, else that block is evaluated
// exactly in fp32), and dS = (K * exp(b_C - b))^T V.
#pragma once

namespace gtr {
namespace pp {

constexpr int kDK = 64;
constexpr int kNStage = 3;                   // staging slots
constexpr int kRing = 3;                     // chunks of a later span whose Qint * D_c stays in smem
constexpr int kMaxSpan = 32;                 // chunks of a span with recorded decays (P > 1)
constexpr int kThreads = 576;                // 18 warps
constexpr int kWarpProd = 0, kWarpMMA = 1, kWarpU = 2, kWarpRE = 6, kWarpG = 10;
constexpr int kUThreads = 128, kREThreads = 128, kGThreads = 256;
constexpr uint32_t kBarG = 1, kBarU = 2, kBarRE = 3, kBarUP = 4, kBarT0 = 5, kBarT1 = 6;
constexpr int kAggFloats = kDK * kDV + kDK;  // state + decay product
constexpr int kAggBytes = kAggFloats * 4;    // 16640
constexpr int kFoldSlots = 8;                // aggregates copied into smem at a time
constexpr int kFlagStride = 32;              // one 128-byte line per publish flag
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kFastMinLogDecay = -6.f;     // fast path: chunk decay >= e^-6
constexpr float kFastMaxK = 100.f;           //            and |k| <= 100
constexpr float kDiagMinLogTotal = -8.f;     // sub-block path: diagonal block decay >= e^-8
constexpr float kDiagMaxK = 30000.f;         //   and |K * e^-bp| stays inside fp16
// TMEM columns: scores [2] x 128 (diagonal / fast scores 0..63, below-diagonal blocks
// 64..111), dS [2] x 64, O [2] x 64
constexpr uint32_t kColScores = 0, kColDS = 256, kColO = 384;
constexpr int kTmemCols = 512;

// ------------------------------------------------------------------ smem map
struct L {
    static constexpr int stage_bytes = 36 * 1024;   // q, k, g, v raw rows + slack
    static constexpr int st_q = 0, st_k = kTile, st_g = 2 * kTile, st_v = 3 * kTile;
    // sub-block operands overlaid on the chunk's staging slot once its raw rows are
    // consumed (the slot is released by MMA 1's completion then):
    //   rows 0..63 Qd, 64..111 A_0, 112..143 A_1, 144..159 A_2 (A_J: rows 16(J+1)..63)
    static constexpr int sl_qa = 0;
    static constexpr int sl_kd = 160 * 128;          // Kd [64][64]
    static constexpr int sl_b = sl_kd + kTile;       // B_J rows 16J..16J+15, J < 3
    static_assert(sl_b + 48 * 128 <= stage_bytes, "sub-block operands fit a staging slot");
    static constexpr int stage = 0;
    static constexpr int qint = stage + kNStage * stage_bytes;   // [2] Qint
    static constexpr int kt = qint + 2 * kTile;                  // [2] K~ (or K^ on the sub-block path)
    static constexpr int vop = kt + 2 * kTile;                   // [2] V in scan order
    static constexpr int sop = vop + 2 * kTile;                  // [2] S_prev fp16
    static constexpr int ring = sop + 2 * kTile;                 // [kRing] Qint * D_c
    static constexpr int ostg = ring + kRing * kTile;            // output staging
    static constexpr int diagx = ostg + kTile;                   // [2][4][16][16] fp16 exact blocks
    static constexpr int dcum = diagx + 2 * 2048;                // [kMaxSpan+1][64] D_c
    static constexpr int dloc = dcum + (kMaxSpan + 1) * 256;     // [2][64] chunk decay d
    static constexpr int htot = dloc + 2 * 256;                  // [8][64] 8-token group totals
    static constexpr int wmax = htot + 8 * 256;                  // [2][16] max |q|, |k| per G warp
    static constexpr int bflag = wmax + 2 * 64;                  // [2][4] exact diagonal blocks
    static constexpr int slowf = bflag + 32;                     // [2] sub-block path
    static constexpr int meta = slowf + 32;                      // [3] staging row table + rows
    static constexpr int rowtab = meta + kNStage * 128;          // [2][64] output token rows
    static constexpr int cmeta = rowtab + 2 * 256;               // [kMaxSpan] max|q|, max|o|
    static constexpr int rmax = cmeta + kMaxSpan * 8;            // [64] row maxima of |S_in|
    static constexpr int work = rmax + 256;                      // [kMaxSpan] phase-4 work list
    static constexpr int bars = work + kMaxSpan * 4 + 16;
    static constexpr int nbars = 32;
    static constexpr int tslot = bars + nbars * 8;
    static constexpr int bytes = tslot + 16;
    static constexpr int alloc = bytes + 1024;
    // after the chunk pipeline: aggregate slots for the look-back
    static constexpr int slots = 0;
    static_assert(kFoldSlots * kAggBytes <= sop, "look-back slots below the S_in operand tile");
};
static_assert(L::alloc <= 227 * 1024, "shared memory budget");
static_assert(L::dcum % 16 == 0 && L::htot % 16 == 0 && L::meta % 16 == 0 && L::rowtab % 16 == 0 &&
                  L::bars % 8 == 0 && L::wmax % 16 == 0,
              "misc alignment");
static_assert(L::qint % 1024 == 0 && L::ring % 1024 == 0 && L::ostg % 1024 == 0, "tile alignment");

enum {
    B_FULL = 0,     // [3] staging slot landed (TMA transaction count)
    B_EMPTY = 3,    // [3] staging slot free again (G, or MMA 1 on the sub-block path)
    B_OPFULL = 6,   // [2] G done: Qint, K~, V, d, flags of a chunk
    B_MMA1 = 8,     // [2] MMA 1 complete
    B_PREADY = 10,  // [2] P written to tensor memory (RE, 128 arrivals)
    B_SPFULL = 12,  // [2] S_prev operand written (U)
    B_MMA2 = 14,    // [2] MMA 2 complete (operands, S_prev, scores free; O ready)
    B_DSFREE = 16,  // [2] dS read by U (128 arrivals)
    B_OFREE = 18,   // [2] O read by RE (128 arrivals)
    B_AGG = 20,     // look-back aggregates copied
    B_FIX = 21,     // correction MMAs complete
    B_DRAIN = 22    // every MMA of the sequence's chunks complete (one phase per sequence)
};

struct Maps {
    CUtensorMap m[4][7];   // q, k, g, v x box heights 64, 32, .., 1 (index = log2 height)
};

struct Args {
    Maps maps;
    Params P;
    float *ws;          // [n_seq][PS][kAggFloats]
    unsigned *flags;    // [n_seq][PS] publish flags, kFlagStride apart
    int PS, Lc;
    unsigned used;      // bit h: the maps of box height 2^h are encoded
    float inv_tau;      // gate-from-z kernel: 1 / tau
};

__device__ __forceinline__ uint64_t *bar(uint8_t *sm, int i) {
    return reinterpret_cast<uint64_t *>(sm + L::bars) + i;
}
__device__ __forceinline__ void wait_l(uint64_t *b, uint32_t parity, bool &to) {
    if (to) return;
    if (!mbar_wait_bounded(b, parity, kWaitLimitNs)) {
        to = true;
        set_error(kErrTimeout);
    }
}
__device__ __forceinline__ float ex2a(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ __half2 h2(float a, float b) { return __floats2half2_rn(a, b); }
// A value about to become an fp16 operand or output must be finite and below 65504.
__device__ __forceinline__ void range_check(float mx) {
    if (!(mx <= kHalfMax)) set_error(kErrRange);
}
template <int N>
__device__ __forceinline__ float max_abs(const float (&x)[N]) {
    float m = 0.f;
#pragma unroll
    for (int e = 0; e < N; ++e) m = fmaxf(m, fabsf(x[e]));
    return m;
}
__device__ __forceinline__ void sth2(uint8_t *p, __half2 v) { *reinterpret_cast<__half2 *>(p) = v; }

__device__ __forceinline__ void tma_4d(uint32_t dst, const CUtensorMap *m, int c0, int c1, int c2, int c3,
                                       uint32_t mbar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, "
        "%4, %5}], [%6];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(mbar)
        : "memory");
}
__device__ __forceinline__ void tma_5d(uint32_t dst, const CUtensorMap *m, int c0, int c1, int c2, int c3, int c4,
                                       uint32_t mbar) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, "
        "%4, %5, %6}], [%7];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(mbar)
        : "memory");
}
__device__ __forceinline__ void tma_prefetch_4d(const CUtensorMap *m, int c0, int c1, int c2, int c3) {
    asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];" ::"l"(
                     reinterpret_cast<uint64_t>(m)),
                 "r"(c0), "r"(c1), "r"(c2), "r"(c3)
                 : "memory");
}
__device__ __forceinline__ void tma_prefetch_5d(const CUtensorMap *m, int c0, int c1, int c2, int c3, int c4) {
    asm volatile("cp.async.bulk.prefetch.tensor.5d.L2.global.tile [%0, {%1, %2, %3, %4, %5}];" ::"l"(
                     reinterpret_cast<uint64_t>(m)),
                 "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
                 : "memory");
}

// 16 TMEM lanes x 256 bit, 2 repeats (16 columns)
__device__ __forceinline__ void tmem_ld_16x256b_x2(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.16x256b.x2.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7])
                 : "r"(taddr)
                 : "memory");
}
__device__ __forceinline__ void tmem_st_16x128b_x8(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.16x128b.x8.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

// Log-decay of the key-side forget gate from its pre-activation z (GTR news article,
// section "线性注意力到底在省什么"): g = log(sigmoid(z)) / tau = (min(z, 0) - log(1 + e^-|z|))
// / tau, with CUDA's exp / log intrinsics (relative error ~2^-21, far below the fp16
// rounding of z itself; for |z| > 17 the log term falls below fp32's resolution of 1 + x,
// an absolute error under 1e-7 / tau).
__device__ __forceinline__ float gate_of(float z, float inv_tau) {
    return (fminf(z, 0.f) - __logf(1.f + __expf(-fabsf(z)))) * inv_tau;
}
template <bool kZ>
__device__ __forceinline__ float2 ld_gate2(const uint8_t *p, float inv_tau) {
    const float2 x = ld_h2(p);
    if constexpr (kZ) return make_float2(gate_of(x.x, inv_tau), gate_of(x.y, inv_tau));
    return x;
}
template <bool kZ>
__device__ __forceinline__ float ld_gate1(const uint8_t *p, float inv_tau) {
    const float x = __half2float(*reinterpret_cast<const __half *>(p));
    if constexpr (kZ) return gate_of(x, inv_tau);
    return x;
}

// ------------------------------------------------------------------ producer
// Staging row table of chunk `cabs` (scan positions p0 .. p0+63): row t of the chunk (in
// scan order) sits at staging row srow[t].  Lanes write two entries each.
__device__ __forceinline__ void write_meta(const Params &P, uint8_t *meta, int cabs, int lane) {
    const int p0 = cabs * kChunk, pend = min(p0 + kChunk, P.N);
    const bool rev = P.dir == GTR_R2L || P.dir == GTR_B2T;
    const int run = P.dir == GTR_R2L ? P.W : P.H;   // run length of a full grid row / column
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int t = lane + 32 * h, p = p0 + t;
        int r = t;
        if (rev && p < pend) {
            const int k = p / run;
            const int lo = max(k * run, p0) - p0, hi = min((k + 1) * run, pend) - 1 - p0;
            r = lo + hi - t;
        }
        meta[t] = (uint8_t)r;
    }
    if (lane == 0) *reinterpret_cast<int *>(meta + 64) = pend - p0;
}

// TMA copies of chunk `cabs` of sequence `seq` into staging slot `slot` (one lane).
// Returns the bytes the copies deliver.
__device__ __forceinline__ uint32_t issue_chunk(const Args &A, uint32_t slot, int seq, int cabs, uint32_t mbar,
                                                bool count_only) {
    const Params &P = A.P;
    const int p0 = cabs * kChunk, pend = min(p0 + kChunk, P.N);
    const int bb = seq / P.heads, hh = seq - bb * P.heads;
    constexpr uint32_t kRowBytes = (3 * kDK + kDV) * 2;
    if (P.dir == GTR_L2R) {
        // one run of 64 tokens; rows past the grid are the copy's zero fill
        if (!count_only)
#pragma unroll
            for (int ten = 0; ten < 4; ++ten)
                tma_4d(slot + ten * kTile, &A.maps.m[ten][6], 0, hh, p0, bb, mbar);
        return 64u * kRowBytes;
    }
    if (!count_only) {
        int p = p0;
        while (p < pend) {
            int len, c2;   // run length, its first coordinate along the run's axis
            int x = 0;
            if (P.dir == GTR_R2L) {
                const int y = p / P.W, q = min((y + 1) * P.W, pend);
                len = q - p;
                c2 = y * P.W + (y + 1) * P.W - q;   // lowest token of the run
            } else {
                x = p / P.H;
                const int q = min((x + 1) * P.H, pend);
                len = q - p;
                c2 = P.dir == GTR_T2B ? p - x * P.H : (x + 1) * P.H - q;   // lowest y of the run
            }
            int off = 0;
            const uint32_t row0 = (uint32_t)(p - p0);
            for (int lb = 6; lb >= 0; --lb) {
                if (!(len & (1 << lb))) continue;
                const uint32_t d = slot + (row0 + off) * 128u;
#pragma unroll
                for (int ten = 0; ten < 4; ++ten) {
                    if (P.dir == GTR_R2L)
                        tma_4d(d + ten * kTile, &A.maps.m[ten][lb], 0, hh, c2 + off, bb, mbar);
                    else
                        tma_5d(d + ten * kTile, &A.maps.m[ten][lb], 0, hh, x, c2 + off, bb, mbar);
                }
                off += 1 << lb;
            }
            p += len;
        }
    }
    return (uint32_t)(pend - p0) * kRowBytes;
}

// ------------------------------------------------------------------ gating (group G)
// G warp gw (0..7) owns scan rows 8gw .. 8gw+7 of the chunk, lane l channels 2l, 2l+1.
struct GRegs {
    __half2 q[8], k[8];
    float2 g[8], p[8];   // log-decays and their prefix sums within the 8-row group
};

// Exact fp32 diagonal blocks of the flagged sub-blocks (rare: decay below e^-8 inside 16
// tokens, or keys too large): value(u, w) = sum_i q[u] k[w] exp(sum_{r=w+1..u} g[r]),
// stored as fp16 (it becomes an fp16 P entry anyway).
template <bool kZ>
__device__ __noinline__ void exact_diag(const uint8_t *st, const uint8_t *meta, int nrows, const int *flags,
                                        __half *dst, int tg, float inv_tau) {
    for (int task = tg; task < 4 * 256; task += kGThreads) {
        const int I = task >> 8, u = (task >> 4) & 15, w = task & 15;
        if (!flags[I] || w > u) continue;
        const int tu = 16 * I + u, tw = 16 * I + w;
        float acc = 0.f;
        if (tu < nrows) {
            const int ru = meta[tu], rw = meta[tw];
            for (int i = 0; i < kDK; ++i) {
                float lg = 0.f;
                for (int r = tw + 1; r <= tu; ++r)
                    lg += ld_gate1<kZ>(st + L::st_g + meta[r] * 128 + 2 * i, inv_tau);
                const float qv = __half2float(*reinterpret_cast<const __half *>(st + L::st_q + ru * 128 + 2 * i));
                const float kv = __half2float(*reinterpret_cast<const __half *>(st + L::st_k + rw * 128 + 2 * i));
                acc += qv * kv * ex2a(lg * kLog2e);
            }
        }
        dst[(I * 16 + u) * 16 + w] = __float2half_rn(acc);
    }
}

// Sub-block path of the gating of one chunk (out of line: the fast path keeps its
// registers).  Writes Qint and K^ = K * exp(b_C - b) into qo / ko (and Qint * D_c into ro
// when held), flags the diagonal blocks that need the exact evaluation, evaluates those
// into diagx[b], then overlays Qd, Kd, A_J and B_J on the chunk's staging slot.
template <bool kZ>
__device__ __noinline__ void gate_slow(uint8_t *sm, const GRegs &R, const float2 (&ht)[8], int gw, int lane, int tg,
                                       uint8_t *st, const uint8_t *meta, int nrows, uint8_t *qo, uint8_t *ko,
                                       uint8_t *ro, bool held, float2 Dc, int *bfl, int b, float inv_tau) {
    const int t0 = 8 * gw;
    const int I = gw >> 1, hb = gw & 1;
    float2 T[4];
#pragma unroll
    for (int J = 0; J < 4; ++J) T[J] = make_float2(ht[2 * J].x + ht[2 * J + 1].x, ht[2 * J].y + ht[2 * J + 1].y);
    float2 pre = make_float2(0.f, 0.f), post = make_float2(0.f, 0.f);
#pragma unroll
    for (int J = 0; J < 4; ++J) {
        if (J < I) { pre.x += T[J].x; pre.y += T[J].y; }
        if (J > I) { post.x += T[J].x; post.y += T[J].y; }
    }
    const float2 poff = hb ? ht[gw - 1] : make_float2(0.f, 0.f);
    const float2 soff = hb ? make_float2(0.f, 0.f) : ht[gw + 1];
    float2 bs[8];   // within-block suffix sums (excluding the row)
    {
        float2 a = soff;
#pragma unroll
        for (int u = 7; u >= 0; --u) {
            bs[u] = a;
            a.x += R.g[u].x;
            a.y += R.g[u].y;
        }
    }
    bool kbad = !(T[I].x >= kDiagMinLogTotal) || !(T[I].y >= kDiagMinLogTotal);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const float2 bp = make_float2(poff.x + R.p[u].x, poff.y + R.p[u].y);
        const float2 qf = __half22float2(R.q[u]), kf = __half22float2(R.k[u]);
        const float2 qi = make_float2(qf.x * ex2a((pre.x + bp.x) * kLog2e), qf.y * ex2a((pre.y + bp.y) * kLog2e));
        const uint32_t o = sw_off(t0 + u, 2 * lane);
        sth2(qo + o, h2(qi.x, qi.y));
        sth2(ko + o, h2(kf.x * ex2a((bs[u].x + post.x) * kLog2e), kf.y * ex2a((bs[u].y + post.y) * kLog2e)));
        if (held) sth2(ro + o, h2(qi.x * Dc.x, qi.y * Dc.y));
        const float kd0 = kf.x * ex2a(-bp.x * kLog2e), kd1 = kf.y * ex2a(-bp.y * kLog2e);
        kbad |= !(fabsf(kd0) <= kDiagMaxK) || !(fabsf(kd1) <= kDiagMaxK);
    }
    if (__any_sync(0xffffffffu, kbad) && lane == 0) atomicOr(&bfl[I], 1);
    named_sync(kBarG, kGThreads);
    const bool anyflag = (bfl[0] | bfl[1] | bfl[2] | bfl[3]) != 0;
    if (anyflag)
        exact_diag<kZ>(st, meta, nrows, bfl, reinterpret_cast<__half *>(sm + L::diagx + b * 2048), tg, inv_tau);
    named_sync(kBarG, kGThreads);   // raw rows no longer read: overlay the operands
    const bool fl = bfl[I] != 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const int t = t0 + u;
        const float2 bp = make_float2(poff.x + R.p[u].x, poff.y + R.p[u].y);
        const float2 qf = __half22float2(R.q[u]), kf = __half22float2(R.k[u]);
        const float2 e = make_float2(ex2a(bp.x * kLog2e), ex2a(bp.y * kLog2e));
        sth2(st + L::sl_qa + sw_off(t, 2 * lane), h2(qf.x * e.x, qf.y * e.y));
        float kd0 = kf.x * ex2a(-bp.x * kLog2e), kd1 = kf.y * ex2a(-bp.y * kLog2e);
        if (fl) kd0 = kd1 = 0.f;
        sth2(st + L::sl_kd + sw_off(t, 2 * lane), h2(kd0, kd1));
        // A_J rows (J < I): anchor at the end of key block J
        float2 acc = bp;
#pragma unroll
        for (int J = 2; J >= 0; --J) {
            if (J < I) {
                const int reg = (J == 0 ? 64 : J == 1 ? 112 : 144) + t - 16 * (J + 1);
                sth2(st + L::sl_qa + sw_off(reg, 2 * lane),
                     h2(qf.x * ex2a(acc.x * kLog2e), qf.y * ex2a(acc.y * kLog2e)));
                acc.x += T[J].x;   // one more block between row and anchor
                acc.y += T[J].y;
            }
        }
        if (I < 3)   // B_I rows: keys of block I, anchor at its end
            sth2(st + L::sl_b + sw_off(t, 2 * lane),
                 h2(kf.x * ex2a(bs[u].x * kLog2e), kf.y * ex2a(bs[u].y * kLog2e)));
    }
}

// ------------------------------------------------------------------ readout helpers
// TMEM fragment of a 64-row accumulator (M = 64 layout), 64 columns: warp quarter q4 holds
// rows 16 q4 + l/4 (+8); register 16 h + 4 j + 2 e + x is row r0 + 8e, column
// 32 h + 8 j + 2 (l % 4) + x.
__device__ __forceinline__ void ld_acc64(uint32_t taddr, uint32_t (&r)[32]) {
    uint32_t (&a)[16] = *reinterpret_cast<uint32_t(*)[16]>(&r[0]);
    uint32_t (&b)[16] = *reinterpret_cast<uint32_t(*)[16]>(&r[16]);
    tmem_ld_16x256b_x4(taddr, a);
    tmem_ld_16x256b_x4(taddr + 32, b);
}

// Output tile (fp32 in registers, fragment layout) -> fp16 -> staging -> coalesced rows.
// Team of 4 warps (128 threads, named barrier `bid`); returns the thread's max |o|.
__device__ __forceinline__ float store_out_tile(const Params &P, const uint32_t (&r)[32], int q4, int lane, int tb,
                                                uint8_t *os, const int *rows, uint32_t bid) {
    const int r0 = 16 * q4 + (lane >> 2), a2 = 2 * (lane & 3);
    float mx = 0.f;
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
        const int h = e >> 4, j = (e >> 2) & 3, hh = (e >> 1) & 1;
        const float x0 = __uint_as_float(r[e]), x1 = __uint_as_float(r[e + 1]);
        mx = fmaxf(mx, fmaxf(fabsf(x0), fabsf(x1)));
        sth2(os + sw_off(r0 + 8 * hh, 32 * h + 8 * j + a2), h2(x0, x1));
    }
    named_sync(bid, 128);
#pragma unroll
    for (int x = tb; x < 64 * 8; x += 128) {
        const int row = x >> 3, c8 = x & 7;
        const int ro = rows[row];
        if (ro >= 0)
            *reinterpret_cast<uint4 *>(P.out + (size_t)ro * kDV + 8 * c8) =
                *reinterpret_cast<const uint4 *>(os + sw_off(row, 8 * c8));
    }
    named_sync(bid, 128);
    return mx;
}

// Correction tile (fp32, fragment layout) added onto the stored fp16 outputs with
// reductions (one addend per element: the result does not depend on their order).
__device__ __forceinline__ void add_out_tile(const Params &P, const uint32_t (&r)[32], int q4, int lane,
                                             const int *rows) {
    const int r0 = 16 * q4 + (lane >> 2), a2 = 2 * (lane & 3);
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
        const int h = e >> 4, j = (e >> 2) & 3, hh = (e >> 1) & 1;
        const int ro = rows[r0 + 8 * hh];
        if (ro < 0) continue;
        const __half2 v = h2(__uint_as_float(r[e]), __uint_as_float(r[e + 1]));
        __half *dst = P.out + (size_t)ro * kDV + 32 * h + 8 * j + a2;
        asm volatile("red.global.add.noftz.f16x2 [%0], %1;" ::"l"(dst), "r"(*reinterpret_cast<const uint32_t *>(&v))
                     : "memory");
    }
}

__device__ __forceinline__ void fill_rowtab(const Params &P, int seq, int cabs, int *rows, int t) {
    if (t < 64) {
        const int p = cabs * kChunk + t;
        int ro = -1;
        if (p < P.N) {
            const int bb = seq / P.heads, hh = seq - bb * P.heads;
            ro = (bb * P.N + scan_to_token(p, P.H, P.W, P.dir)) * P.heads + hh;
        }
        rows[t] = ro;
    }
}

// fp16 copy of a 64x64 fp32 fragment (U's layout) into a swizzled MN-major operand tile.
__device__ __forceinline__ void write_state_tile(uint8_t *dst, const float (&S)[32], int q4, int lane) {
    const int r0 = 16 * q4 + (lane >> 2), a2 = 2 * (lane & 3);
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
        const int h = e >> 4, j = (e >> 2) & 3, hh = (e >> 1) & 1;
        sth2(dst + sw_off(r0 + 8 * hh, 32 * h + 8 * j + a2), h2(S[e], S[e + 1]));
    }
}

// ------------------------------------------------------------------ kernel
// kZ: the third input holds the gate pre-activation z instead of the log-decay g.
template <bool kZ>
__global__ void __launch_bounds__(kThreads, 1) gla_fwd_pipe_kernel(const __grid_constant__ Args A) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    const Params &P = A.P;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int PS = A.PS;
    const int kspan = (int)blockIdx.x % PS;
    const int grp = (int)blockIdx.x / PS, ngrp = (int)gridDim.x / PS;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + L::tslot);
    float *dcum = reinterpret_cast<float *>(sm + L::dcum);
    float *cmeta = reinterpret_cast<float *>(sm + L::cmeta);

    if (warp == kWarpMMA) {
        tmem_alloc(tslot, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < kNStage; ++i) {
            mbar_init(bar(sm, B_FULL + i), 1);
            mbar_init(bar(sm, B_EMPTY + i), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(sm, B_OPFULL + i), 1);
            mbar_init(bar(sm, B_MMA1 + i), 1);
            mbar_init(bar(sm, B_PREADY + i), kREThreads);
            mbar_init(bar(sm, B_SPFULL + i), 1);
            mbar_init(bar(sm, B_MMA2 + i), 1);
            mbar_init(bar(sm, B_DSFREE + i), kUThreads);
            mbar_init(bar(sm, B_OFREE + i), kREThreads);
        }
        mbar_init(bar(sm, B_AGG), 1);
        mbar_init(bar(sm, B_FIX), 1);
        mbar_init(bar(sm, B_DRAIN), 1);
        fence_mbar_init();
    }
    if (warp == kWarpProd && lane < 28 && (lane & 7) < 7 && ((A.used >> (lane & 7)) & 1u))
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&A.maps.m[lane >> 3][lane & 7]))
                     : "memory");
    // the first chunk's rows into L2 while the grid ahead drains (L2 is where every
    // SM's accesses meet, so a later write by that grid still reaches the copies)
    if (warp == kWarpProd && lane == 0 && grp < P.n_seq && P.dir == GTR_L2R) {
        const int seq = grp, bb = seq / P.heads, hh = seq - bb * P.heads;
        const int c0 = kspan * A.Lc;
        for (int ten = 0; ten < 4; ++ten) tma_prefetch_4d(&A.maps.m[ten][6], 0, hh, c0 * kChunk, bb);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    bool to = false;
    uint32_t gc0 = 0;          // chunks of earlier sequences run by this CTA
    uint32_t n_agg = 0, n_fix = 0, n_drain = 0;

    for (int seq = grp; seq < P.n_seq; seq += ngrp) {
        const int c0 = kspan * A.Lc;
        const int nch = min(A.Lc, P.n_chunks - c0);   // >= 1 (host guarantees)
        const bool later = kspan > 0;
        const bool publish = PS > 1 && kspan < PS - 1;
        const int nring = later ? min(kRing, nch) : 0;

        if (warp == kWarpProd) {
            // ======================================================= producer
            for (int c = 0; c < nch; ++c) {
                const uint32_t gc = gc0 + c, s = gc % kNStage;
                wait_l(bar(sm, B_EMPTY + s), ((gc / kNStage) & 1u) ^ 1u, to);
                write_meta(P, sm + L::meta + s * 128, c0 + c, lane);
                __syncwarp();
                if (lane == 0) {
                    const uint32_t mb = smem_u32(bar(sm, B_FULL + s));
                    const uint32_t slot = sbase + L::stage + s * L::stage_bytes;
                    mbar_arrive_expect_tx(bar(sm, B_FULL + s), issue_chunk(A, slot, seq, c0 + c, mb, true));
                    issue_chunk(A, slot, seq, c0 + c, mb, false);
                }
                __syncwarp();
            }
            // Every MMA of this sequence's chunks complete (their operand tiles are free).
            // A dedicated barrier with one phase per sequence: this warp runs ahead of the
            // pipeline, so a parity wait on a per-buffer barrier could match an earlier phase.
            wait_l(bar(sm, B_DRAIN), n_drain & 1u, to);
            ++n_drain;
            if (later) {
                // ---------------- phase 3: the earlier spans' aggregates into shared memory.
                // The slots overlay the staging ring and the first operand tiles (free now).
                // Lane u polls span j0+u's flag and copies that aggregate at once; group U
                // folds a batch, then releases the slots (named barrier kBarUP).
                for (int j0 = 0; j0 < kspan; j0 += kFoldSlots) {
                    const int nj = min(kFoldSlots, kspan - j0);
                    if (lane == 0) mbar_arrive_expect_tx(bar(sm, B_AGG), (uint32_t)(nj * kAggBytes));
                    __syncwarp();
                    if (lane < nj) {
                        unsigned *f = A.flags + ((size_t)seq * PS + j0 + lane) * kFlagStride;
                        if (sp::flag_wait_bounded(f, kWaitLimitNs)) {
                            sp::red_dec_gpu(f);   // one reader fewer to come
                        } else {
                            to = true;
                            set_error(kErrTimeout);
                        }
                        // the copy engine reads what the acquire made visible; after a
                        // timeout the copy still runs, so that the barrier completes
                        asm volatile("fence.proxy.async.global;" ::: "memory");
                        bulk_g2s(sbase + L::slots + lane * kAggBytes,
                                 A.ws + ((size_t)seq * PS + j0 + lane) * kAggFloats, (uint32_t)kAggBytes,
                                 bar(sm, B_AGG));
                    }
                    named_sync(kBarUP, kUThreads + 32);   // U done with the slots
                }
            }
        } else if (warp == kWarpMMA) {
            // ======================================================= MMA issuer
            constexpr uint32_t id_ds = idesc_f16_f32(64, kDV, true, true);
            constexpr uint32_t id_sc = idesc_f16_f32(64, 64, false, false);
            constexpr uint32_t id_off = idesc_f16_f32(64, 16, false, false);
            constexpr uint32_t id_o = idesc_f16_f32(64, kDV, false, true);
            // Issues MMA 1 of the next chunk or MMA 2 of the oldest chunk, whichever has its
            // inputs first (MMA 1 of chunk c also needs MMA 2 of chunk c-2 complete, so it
            // never runs more than one chunk ahead).  Each barrier's phases are tested in
            // order, one at a time, so a test can never match an earlier phase.
            int n1 = 0, n2 = 0;
            long long idle0 = cycles();
            while (n2 < nch) {
                bool did = false;
                if (n1 < nch && n1 <= n2 + 1) {
                    const uint32_t gc = gc0 + n1, b = gc & 1u, s = gc % kNStage, ph = (gc >> 1) & 1u;
                    const bool ready = to || (mbar_test(bar(sm, B_OPFULL + b), ph) &&
                                              (gc < 2 || (mbar_test(bar(sm, B_DSFREE + b), ph ^ 1u) &&
                                                          mbar_test(bar(sm, B_MMA2 + b), ph ^ 1u))));
                    if (__all_sync(0xffffffffu, ready)) {
                        tc_fence_after();
                        const bool slow = reinterpret_cast<const int *>(sm + L::slowf)[b] != 0;
                        const uint32_t kta = sbase + L::kt + b * kTile, va = sbase + L::vop + b * kTile;
                        const uint32_t qa = sbase + L::qint + b * kTile;
                        const uint32_t sl = sbase + L::stage + s * L::stage_bytes;
                        const uint32_t dsc = tmem + kColDS + 64 * b, scc = tmem + kColScores + 128 * b;
                        if (elect_one_sync()) {
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                umma_f16(dsc, desc_sw128(kta + kk * 2048, kTile, 1024),
                                         desc_sw128(va + kk * 2048, kTile, 1024), id_ds, kk > 0 ? 1u : 0u);
                            if (!slow) {
#pragma unroll
                                for (int kk = 0; kk < 4; ++kk)
                                    umma_f16(scc, desc_sw128(qa + kk * 32, 16, 1024),
                                             desc_sw128(kta + kk * 32, 16, 1024), id_sc, kk > 0 ? 1u : 0u);
                            } else {
#pragma unroll
                                for (int kk = 0; kk < 4; ++kk)
                                    umma_f16(scc, desc_sw128(sl + L::sl_qa + kk * 32, 16, 1024),
                                             desc_sw128(sl + L::sl_kd + kk * 32, 16, 1024), id_sc, kk > 0 ? 1u : 0u);
                                // A_J's descriptor starts 16(J+1) rows before its region, so that
                                // row t of the operand is scan row t (earlier rows: finite values of
                                // the regions before it, whose results are never read)
                                const uint32_t abase[3] = {48u * 128u, 80u * 128u, 96u * 128u};
#pragma unroll
                                for (int J = 0; J < 3; ++J)
#pragma unroll
                                    for (int kk = 0; kk < 4; ++kk)
                                        umma_f16(scc + 64 + 16 * J,
                                                 desc_sw128(sl + L::sl_qa + abase[J] + kk * 32, 16, 1024),
                                                 desc_sw128(sl + L::sl_b + J * 2048 + kk * 32, 16, 1024), id_off,
                                                 kk > 0 ? 1u : 0u);
                            }
                            umma_commit(bar(sm, B_MMA1 + b));
                            if (slow) umma_commit(bar(sm, B_EMPTY + s));   // the overlaid slot is free
                        }
                        __syncwarp();
                        ++n1;
                        did = true;
                    }
                }
                if (!did && n2 < n1) {
                    const uint32_t gp = gc0 + n2, b = gp & 1u, ph = (gp >> 1) & 1u;
                    const bool ready = to || (mbar_test(bar(sm, B_PREADY + b), ph) &&
                                              mbar_test(bar(sm, B_SPFULL + b), ph) &&
                                              (gp < 2 || mbar_test(bar(sm, B_OFREE + b), ph ^ 1u)));
                    if (__all_sync(0xffffffffu, ready)) {
                        tc_fence_after();
                        const uint32_t qa = sbase + L::qint + b * kTile, sa = sbase + L::sop + b * kTile;
                        const uint32_t va = sbase + L::vop + b * kTile;
                        const uint32_t oc = tmem + kColO + 64 * b, pc = tmem + kColScores + 128 * b;
                        if (elect_one_sync()) {
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                umma_f16(oc, desc_sw128(qa + kk * 32, 16, 1024),
                                         desc_sw128(sa + kk * 2048, kTile, 1024), id_o, kk > 0 ? 1u : 0u);
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)   // P from TMEM: K step 16 = 8 packed columns
                                umma_f16_ta(oc, pc + 8 * kk, desc_sw128(va + kk * 2048, kTile, 1024), id_o, 1u);
                            umma_commit(bar(sm, B_MMA2 + b));
                            if (n2 + 1 == nch) umma_commit(bar(sm, B_DRAIN));   // the sequence's last MMA
                        }
                        __syncwarp();
                        ++n2;
                        did = true;
                    }
                }
                if (did) {
                    idle0 = cycles();
                } else if (cycles() - idle0 <= cycles_of_ns(kWaitLimitNs)) {
                    __nanosleep(16);   // leave the issue slots to the warps doing the work
                } else {
                    if (!to) set_error(kErrTimeout);
                    to = true;   // from now on every test passes: the kernel runs to its end
                }
            }
        } else if (warp < kWarpRE) {
            // ======================================================= state group U
            const int q4 = warp & 3, ut = tid - kWarpU * 32;
            const int r0 = 16 * q4 + (lane >> 2);
            float S[32];
            {
                const float *s0 = (!later && P.s0 != nullptr) ? P.s0 + (size_t)seq * kDK * kDV : nullptr;
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const int h = e >> 4, j = (e >> 2) & 3, hh = (e >> 1) & 1;
                    float2 v = make_float2(0.f, 0.f);
                    if (s0) v = *reinterpret_cast<const float2 *>(s0 + (r0 + 8 * hh) * kDV + 32 * h + 8 * j + 2 * (lane & 3));
                    S[e] = v.x;
                    S[e + 1] = v.y;
                }
            }
            // S_prev of the first chunk; then (for the next chunk's d and flags, and so
            // that G cannot complete that buffer's next phase before this wait) G's signal
            float dn0, dn1;
            bool slown;
            {
                const uint32_t gn = gc0, bn = gn & 1u, ph = (gn >> 1) & 1u;
                if (gn >= 2) wait_l(bar(sm, B_MMA2 + bn), ph ^ 1u, to);
                range_check(max_abs(S));
                write_state_tile(sm + L::sop + bn * kTile, S, q4, lane);
                fence_proxy_async_cta();
                named_sync(kBarU, kUThreads);
                wait_l(bar(sm, B_OPFULL + bn), ph, to);
                const float *dl = reinterpret_cast<const float *>(sm + L::dloc + bn * 256);
                dn0 = dl[r0];
                dn1 = dl[r0 + 8];
                slown = reinterpret_cast<const int *>(sm + L::slowf)[bn] != 0;
                if (ut == 0) mbar_arrive(bar(sm, B_SPFULL + bn));
            }
            for (int c = 0; c < nch; ++c) {
                const uint32_t gc = gc0 + c, b = gc & 1u, ph = (gc >> 1) & 1u;
                const float d0 = dn0, d1 = dn1;
                const bool slow = slown;
                wait_l(bar(sm, B_MMA1 + b), ph, to);
                tc_fence_after();
                uint32_t ds[32];
                ld_acc64(tmem + ((uint32_t)(32 * q4) << 16) + kColDS + 64 * b, ds);
                tmem_ld_wait();
                tc_fence_before();
                mbar_arrive(bar(sm, B_DSFREE + b));
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const float d = ((e >> 1) & 1) ? d1 : d0;
                    const float x = __uint_as_float(ds[e]);
                    S[e] = slow ? fmaf(d, S[e], x) : d * (S[e] + x);
                }
                if (c + 1 < nch) {
                    const uint32_t gn = gc + 1, bn = gn & 1u, phn = (gn >> 1) & 1u;
                    if (gn >= 2) wait_l(bar(sm, B_MMA2 + bn), phn ^ 1u, to);
                    range_check(max_abs(S));
                    write_state_tile(sm + L::sop + bn * kTile, S, q4, lane);
                    fence_proxy_async_cta();
                    named_sync(kBarU, kUThreads);
                    wait_l(bar(sm, B_OPFULL + bn), phn, to);
                    const float *dl = reinterpret_cast<const float *>(sm + L::dloc + bn * 256);
                    dn0 = dl[r0];
                    dn1 = dl[r0 + 8];
                    slown = reinterpret_cast<const int *>(sm + L::slowf)[bn] != 0;
                    if (ut == 0) mbar_arrive(bar(sm, B_SPFULL + bn));
                }
            }
            if (publish) {
                // aggregate = (state reached from zero, decay product of the span), fragment
                // order: float4 m*128 + q4*32 + lane holds S[4m .. 4m+3] of that thread
                float *agg = A.ws + ((size_t)seq * PS + kspan) * kAggFloats;
                float4 *a4 = reinterpret_cast<float4 *>(agg);
#pragma unroll
                for (int m = 0; m < 8; ++m)
                    a4[m * 128 + q4 * 32 + lane] = make_float4(S[4 * m], S[4 * m + 1], S[4 * m + 2], S[4 * m + 3]);
                // (dcum[nch] was written by G before its signal of the span's last chunk,
                // which this group waited for)
                if (ut < 64) agg[kDK * kDV + ut] = dcum[nch * 64 + ut];
                named_sync(kBarU, kUThreads);
                if (ut == 0)   // readers to come: spans kspan+1 .. PS-1
                    sp::st_release_gpu(A.flags + ((size_t)seq * PS + kspan) * kFlagStride, (unsigned)(PS - 1 - kspan));
            }
            if (PS == 1 && P.sf != nullptr) {
                float *sf = P.sf + (size_t)seq * kDK * kDV;
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const int h = e >> 4, j = (e >> 2) & 3, hh = (e >> 1) & 1;
                    *reinterpret_cast<float2 *>(sf + (r0 + 8 * hh) * kDV + 32 * h + 8 * j + 2 * (lane & 3)) =
                        make_float2(S[e], S[e + 1]);
                }
            }
            // the last span parks its local state in its own (never published) aggregate
            // slot while the look-back runs (not in final_state: with an in-place carry that
            // is span 0's initial state); phase 3 reads back this thread's own elements
            float4 *park = reinterpret_cast<float4 *>(A.ws + ((size_t)seq * PS + kspan) * kAggFloats);
            if (later && kspan == PS - 1 && P.sf != nullptr) {
#pragma unroll
                for (int m = 0; m < 8; ++m)
                    park[m * 128 + q4 * 32 + lane] = make_float4(S[4 * m], S[4 * m + 1], S[4 * m + 2], S[4 * m + 3]);
            }
            if (later) {
                // ---------------- phase 3: look back over spans 0 .. kspan-1
                float Sin[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) Sin[e] = 0.f;
                for (int j0 = 0; j0 < kspan; j0 += kFoldSlots) {
                    const int nj = min(kFoldSlots, kspan - j0);
                    wait_l(bar(sm, B_AGG), n_agg & 1u, to);
                    ++n_agg;
                    for (int u = 0; u < nj; ++u) {   // S_in <- D_j * S_in + S_j
                        const float *a = reinterpret_cast<const float *>(sm + L::slots + u * kAggBytes);
                        const float D0 = a[kDK * kDV + r0], D1 = a[kDK * kDV + r0 + 8];
#pragma unroll
                        for (int m = 0; m < 8; ++m) {
                            const float4 v = reinterpret_cast<const float4 *>(a)[m * 128 + q4 * 32 + lane];
                            Sin[4 * m] = fmaf(D0, Sin[4 * m], v.x);
                            Sin[4 * m + 1] = fmaf(D0, Sin[4 * m + 1], v.y);
                            Sin[4 * m + 2] = fmaf(D1, Sin[4 * m + 2], v.z);
                            Sin[4 * m + 3] = fmaf(D1, Sin[4 * m + 3], v.w);
                        }
                    }
                    named_sync(kBarUP, kUThreads + 32);   // slots free for the next batch
                }
                // row maxima of |S_in| (rows r0: elements 4m, 4m+1; r0 + 8: 4m+2, 4m+3)
                float m0 = 0.f, m1 = 0.f;
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    m0 = fmaxf(m0, fmaxf(fabsf(Sin[4 * m]), fabsf(Sin[4 * m + 1])));
                    m1 = fmaxf(m1, fmaxf(fabsf(Sin[4 * m + 2]), fabsf(Sin[4 * m + 3])));
                }
#pragma unroll
                for (int o = 1; o <= 2; o <<= 1) {
                    m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, o));
                    m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
                }
                float *rmax = reinterpret_cast<float *>(sm + L::rmax);
                if ((lane & 3) == 0) {
                    rmax[r0] = m0;
                    rmax[r0 + 8] = m1;
                }
                // S_in as the fp16 operand of the correction MMAs
                range_check(fmaxf(m0, m1));
                write_state_tile(sm + L::sop, Sin, q4, lane);
                if (kspan == PS - 1 && P.sf != nullptr) {   // final state D_span * S_in + S_local
                    const float G0 = dcum[nch * 64 + r0], G1 = dcum[nch * 64 + r0 + 8];
                    float *sf = P.sf + (size_t)seq * kDK * kDV;
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const int h = e >> 4, j = (e >> 2) & 3, hh = (e >> 1) & 1;
                        const float Gd = hh ? G1 : G0;
                        const float4 pk = park[(e >> 2) * 128 + q4 * 32 + lane];   // S_local[4m .. 4m+3]
                        const float sx = (e & 2) ? pk.z : pk.x, sy = (e & 2) ? pk.w : pk.y;
                        *reinterpret_cast<float2 *>(sf + (r0 + 8 * hh) * kDV + 32 * h + 8 * j + 2 * (lane & 3)) =
                            make_float2(fmaf(Gd, Sin[e], sx), fmaf(Gd, Sin[e + 1], sy));
                    }
                }
                fence_proxy_async_cta();
            }
        } else if (warp < kWarpG) {
            // ======================================================= readout group RE
            const int q4 = warp & 3, rt = tid - kWarpRE * 32;
            const int r0 = 16 * q4 + (lane >> 2), a2 = 2 * (lane & 3);
            for (int c = 0; c <= nch; ++c) {
                if (c < nch) {
                    const uint32_t gc = gc0 + c, b = gc & 1u, ph = (gc >> 1) & 1u;
                    int *rows = reinterpret_cast<int *>(sm + L::rowtab) + 64 * b;
                    fill_rowtab(P, seq, c0 + c, rows, rt);
                    if (rt == 0 && c < kMaxSpan) cmeta[2 * c + 1] = 0.f;
                    wait_l(bar(sm, B_OPFULL + b), ph, to);
                    wait_l(bar(sm, B_MMA1 + b), ph, to);
                    tc_fence_after();
                    const bool slow = reinterpret_cast<const int *>(sm + L::slowf)[b] != 0;
                    const uint32_t ta = tmem + ((uint32_t)(32 * q4) << 16) + kColScores + 128 * b;
                    uint32_t sc[32];
                    ld_acc64(ta, sc);
                    uint32_t pv[16];
                    float pmx = 0.f;
                    if (!slow) {
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            const int h = e >> 4, j = (e >> 2) & 3, hh = (e >> 1) & 1;
                            const int row = r0 + 8 * hh, col = 32 * h + 8 * j + a2;
                            const float x0 = col <= row ? __uint_as_float(sc[e]) : 0.f;
                            const float x1 = col + 1 <= row ? __uint_as_float(sc[e + 1]) : 0.f;
                            pmx = fmaxf(pmx, fmaxf(fabsf(x0), fabsf(x1)));
                            const __half2 v = h2(x0, x1);
                            pv[2 * (j + 4 * h) + hh] = *reinterpret_cast<const uint32_t *>(&v);
                        }
                    } else {
                        uint32_t of[32];
#pragma unroll
                        for (int e = 24; e < 32; ++e) of[e] = 0u;   // key block 3: never below the diagonal
                        {
                            uint32_t (&oa)[16] = *reinterpret_cast<uint32_t(*)[16]>(&of[0]);
                            uint32_t (&ob)[8] = *reinterpret_cast<uint32_t(*)[8]>(&of[16]);
                            tmem_ld_16x256b_x4(ta + 64, oa);
                            tmem_ld_16x256b_x2(ta + 96, ob);
                        }
                        tmem_ld_wait();
                        const int *fl = reinterpret_cast<const int *>(sm + L::bflag) + 4 * b;
                        const bool exact = fl[q4] != 0;
                        const __half *dx = reinterpret_cast<const __half *>(sm + L::diagx + b * 2048) + q4 * 256;
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            const int h = e >> 4, j = (e >> 2) & 3, hh = (e >> 1) & 1;
                            const int row = r0 + 8 * hh, col = 32 * h + 8 * j + a2;
                            const int J = col >> 4;   // key block (col and col + 1 share it)
                            float x0 = 0.f, x1 = 0.f;
                            if (J < q4) {
                                x0 = __uint_as_float(of[e]);
                                x1 = __uint_as_float(of[e + 1]);
                            } else if (J == q4) {
                                if (exact) {
                                    x0 = __half2float(dx[(row & 15) * 16 + (col & 15)]);
                                    x1 = __half2float(dx[(row & 15) * 16 + ((col + 1) & 15)]);
                                } else {
                                    x0 = __uint_as_float(sc[e]);
                                    x1 = __uint_as_float(sc[e + 1]);
                                }
                                x0 = col <= row ? x0 : 0.f;
                                x1 = col + 1 <= row ? x1 : 0.f;
                            }
                            pmx = fmaxf(pmx, fmaxf(fabsf(x0), fabsf(x1)));
                            const __half2 v = h2(x0, x1);
                            pv[2 * (j + 4 * h) + hh] = *reinterpret_cast<const uint32_t *>(&v);
                        }
                    }
                    range_check(pmx);
                    tmem_st_16x128b_x8(ta, pv);
                    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                    tc_fence_before();
                    mbar_arrive(bar(sm, B_PREADY + b));
                }
                if (c >= 1) {
                    const int cp = c - 1;
                    const uint32_t gp = gc0 + cp, b = gp & 1u, ph = (gp >> 1) & 1u;
                    wait_l(bar(sm, B_MMA2 + b), ph, to);
                    tc_fence_after();
                    uint32_t o[32];
                    ld_acc64(tmem + ((uint32_t)(32 * q4) << 16) + kColO + 64 * b, o);
                    tmem_ld_wait();
                    tc_fence_before();
                    mbar_arrive(bar(sm, B_OFREE + b));
                    const float mx = store_out_tile(P, o, q4, lane, rt, sm + L::ostg,
                                                    reinterpret_cast<const int *>(sm + L::rowtab) + 64 * b, kBarRE);
                    range_check(mx);
                    if (later && cp >= kRing && cp < kMaxSpan) {
                        const unsigned w = __reduce_max_sync(0xffffffffu, __float_as_uint(mx));
                        if (lane == 0) atomicMax(reinterpret_cast<unsigned *>(cmeta + 2 * cp + 1), w);
                    }
                }
            }
        } else {
            // ======================================================= gating group G
            const int gw = warp - kWarpG, tg = tid - kWarpG * 32, t0 = 8 * gw;
            float *htot = reinterpret_cast<float *>(sm + L::htot);
            if (tg < 64) dcum[tg] = 1.f;
            for (int c = 0; c < nch; ++c) {
                const uint32_t gc = gc0 + c, b = gc & 1u, s = gc % kNStage, ph = (gc >> 1) & 1u;
                const bool held = c < nring;
                wait_l(bar(sm, B_FULL + s), (gc / kNStage) & 1u, to);
                if (gc >= 2) wait_l(bar(sm, B_MMA2 + b), ph ^ 1u, to);   // operand buffers b free
                uint8_t *st = sm + L::stage + s * L::stage_bytes;
                const uint8_t *meta = sm + L::meta + s * 128;
                const int nrows = *reinterpret_cast<const int *>(meta + 64);
                unsigned *wm = reinterpret_cast<unsigned *>(sm + L::wmax) + 16 * b;
                int *bfl = reinterpret_cast<int *>(sm + L::bflag) + 4 * b;
                if (tg < 4) bfl[tg] = 0;
                // ---------- pass 1: raw rows -> registers, group prefix sums, maxima, V copy
                GRegs R;
                {
                    const uint2 sr = *reinterpret_cast<const uint2 *>(meta + t0);
                    __half2 qm = __float2half2_rn(0.f), km = qm;
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int r = ((u < 4 ? sr.x : sr.y) >> (8 * (u & 3))) & 0xff;
                        const uint32_t o = r * 128 + 4 * lane;
                        if (t0 + u < nrows) {
                            R.g[u] = ld_gate2<kZ>(st + L::st_g + o, A.inv_tau);
                            R.q[u] = *reinterpret_cast<const __half2 *>(st + L::st_q + o);
                            R.k[u] = *reinterpret_cast<const __half2 *>(st + L::st_k + o);
                        } else {
                            R.g[u] = make_float2(0.f, 0.f);
                            R.q[u] = __float2half2_rn(0.f);
                            R.k[u] = R.q[u];
                        }
                        qm = __hmax2(qm, __habs2(R.q[u]));
                        km = __hmax2(km, __habs2(R.k[u]));
                    }
                    float2 acc = make_float2(0.f, 0.f);
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        acc.x += R.g[u].x;
                        acc.y += R.g[u].y;
                        R.p[u] = acc;
                    }
                    *reinterpret_cast<float2 *>(htot + gw * 64 + 2 * lane) = acc;
                    const unsigned wq = __reduce_max_sync(0xffffffffu, __float_as_uint(fmaxf(__low2float(qm), __high2float(qm))));
                    const unsigned wk = __reduce_max_sync(0xffffffffu, __float_as_uint(fmaxf(__low2float(km), __high2float(km))));
                    if (lane == 0) {
                        wm[gw] = wq;
                        wm[8 + gw] = wk;
                    }
                    // V rows into the scan-ordered operand tile: row tg/4, 16-byte pieces
                    // 2 (tg%4), +1
                    {
                        const int t = tg >> 2, pc = 2 * (tg & 3);
                        const int r = meta[t];
                        uint4 v0 = make_uint4(0u, 0u, 0u, 0u), v1 = v0;
                        if (t < nrows) {
                            v0 = *reinterpret_cast<const uint4 *>(st + L::st_v + r * 128 + 16 * pc);
                            v1 = *reinterpret_cast<const uint4 *>(st + L::st_v + r * 128 + 16 * pc + 16);
                        }
                        uint8_t *vo = sm + L::vop + b * kTile;
                        *reinterpret_cast<uint4 *>(vo + sw_off(t, 8 * pc)) = v0;
                        *reinterpret_cast<uint4 *>(vo + sw_off(t, 8 * pc + 8)) = v1;
                    }
                }
                named_sync(kBarG, kGThreads);
                // ---------- pass 2
                float2 ht[8];
#pragma unroll
                for (int w = 0; w < 8; ++w) ht[w] = *reinterpret_cast<const float2 *>(htot + w * 64 + 2 * lane);
                float2 off = make_float2(0.f, 0.f), bC = make_float2(0.f, 0.f);
#pragma unroll
                for (int w = 0; w < 8; ++w) {
                    if (w < gw) {
                        off.x += ht[w].x;
                        off.y += ht[w].y;
                    }
                    bC.x += ht[w].x;
                    bC.y += ht[w].y;
                }
                unsigned kmx = 0u, qmx = 0u;
#pragma unroll
                for (int w = 0; w < 8; ++w) {
                    qmx = max(qmx, wm[w]);
                    kmx = max(kmx, wm[8 + w]);
                }
                const bool bad = !(bC.x >= kFastMinLogDecay) || !(bC.y >= kFastMinLogDecay) ||
                                 __uint_as_float(kmx) > kFastMaxK;
                // every warp's lanes cover all 64 channels: a warp vote is the chunk's decision
                const bool slow = __any_sync(0xffffffffu, bad);
                const float2 Dc = *reinterpret_cast<const float2 *>(dcum + (held ? c : 0) * 64 + 2 * lane);
                uint8_t *qo = sm + L::qint + b * kTile;
                uint8_t *ko = sm + L::kt + b * kTile;
                uint8_t *ro = sm + L::ring + (held ? c : 0) * kTile;
                if (!slow) {
                    if (tg == 0) mbar_arrive(bar(sm, B_EMPTY + s));   // raw rows consumed
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const float x0 = (off.x + R.p[u].x) * kLog2e, x1 = (off.y + R.p[u].y) * kLog2e;
                        const float e0 = ex2a(x0), e1 = ex2a(x1);
                        const __half2 qi = __hmul2(R.q[u], h2(e0, e1));
                        const uint32_t o = sw_off(t0 + u, 2 * lane);
                        sth2(qo + o, qi);
                        sth2(ko + o, __hmul2(R.k[u], h2(ex2a(-x0), ex2a(-x1))));
                        if (held) {   // Qint * D_c in fp32, one rounding
                            const float2 qf = __half22float2(R.q[u]);
                            sth2(ro + o, h2(qf.x * e0 * Dc.x, qf.y * e1 * Dc.y));
                        }
                    }
                } else {
                    gate_slow<kZ>(sm, R, ht, gw, lane, tg, st, meta, nrows, qo, ko, ro, held, Dc, bfl, b, A.inv_tau);
                }
                // chunk decay and decay products from the span start
                if (gw == 0) {
                    const float2 d = make_float2(ex2a(bC.x * kLog2e), ex2a(bC.y * kLog2e));
                    *reinterpret_cast<float2 *>(sm + L::dloc + b * 256 + 8 * lane) = d;
                    if (c < kMaxSpan) {
                        const float2 dc = *reinterpret_cast<const float2 *>(dcum + c * 64 + 2 * lane);
                        *reinterpret_cast<float2 *>(dcum + (c + 1) * 64 + 2 * lane) = make_float2(dc.x * d.x, dc.y * d.y);
                    }
                    if (lane == 0 && c < kMaxSpan) cmeta[2 * c] = __uint_as_float(qmx);
                }
                fence_proxy_async_cta();
                named_sync(kBarG, kGThreads);
                if (tg == 0) {
                    reinterpret_cast<int *>(sm + L::slowf)[b] = slow ? 1 : 0;
                    mbar_arrive(bar(sm, B_OPFULL + b));
                }
            }
        }
        gc0 += (uint32_t)nch;
        __syncthreads();

        if (later) {
            __syncthreads();   // S_in operand, row maxima, final state written
            // ---------------- phase 4: the S_in term (Qint * D_c) S_in of every chunk
            // chunks past the ring: is the term negligible?  |term| <= max|q| *
            // sum_i D_c[i] max_j |S_in[i][j]| (Qint <= |q|), negligible when below 2^-16 of
            // the chunk's largest output.  One warp per chunk.
            int *work = reinterpret_cast<int *>(sm + L::work);
            const float *rmax = reinterpret_cast<const float *>(sm + L::rmax);
            for (int ci = kRing + warp; ci < nch; ci += kThreads / 32) {
                float part = fmaf(dcum[ci * 64 + 2 * lane], rmax[2 * lane], dcum[ci * 64 + 2 * lane + 1] * rmax[2 * lane + 1]);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
                if (lane == 0) work[ci] = !(cmeta[2 * ci] * part <= 1.52587890625e-5f * cmeta[2 * ci + 1]);
            }
            __syncthreads();
            // batches: the ring chunks first, then the rest that need the term, four at a
            // time, their Qint * D_c rebuilt from re-read q and g rows into the free
            // operand tiles (qint[0], qint[1], kt[0], kt[1])
            int next = kRing;
            for (int batch = 0;; ++batch) {
                int list[4];
                int nl = 0;
                uint32_t qaddr[4];
                if (batch == 0) {
                    for (int ci = 0; ci < nring; ++ci) {
                        list[nl] = ci;
                        qaddr[nl] = sbase + L::ring + ci * kTile;
                        ++nl;
                    }
                } else {
                    while (nl < 4 && next < nch) {
                        if (work[next]) {
                            list[nl] = next;
                            qaddr[nl] = sbase + (nl < 2 ? L::qint + nl * kTile : L::kt + (nl - 2) * kTile);
                            ++nl;
                        }
                        ++next;
                    }
                }
                if (nl == 0) {
                    if (batch == 0) continue;
                    break;
                }
                if (batch > 0 && warp >= kWarpG) {
                    // rebuild Qint * D_c of the listed chunks from q and g (plain loads)
                    const int gw = warp - kWarpG, tg = tid - kWarpG * 32, t0 = 8 * gw;
                    float *htot = reinterpret_cast<float *>(sm + L::htot);
                    const int bb = seq / P.heads, hh = seq - bb * P.heads;
                    for (int li = 0; li < nl; ++li) {
                        const int ci = list[li];
                        const int cabs = c0 + ci;
                        __half2 qv[8];
                        float2 pg[8];
                        float2 acc = make_float2(0.f, 0.f);
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const int p = cabs * kChunk + t0 + u;
                            float2 gv = make_float2(0.f, 0.f);
                            qv[u] = __float2half2_rn(0.f);
                            if (p < P.N) {
                                const size_t rowi = ((size_t)bb * P.N + scan_to_token(p, P.H, P.W, P.dir)) * P.heads + hh;
                                gv = ld_gate2<kZ>(reinterpret_cast<const uint8_t *>(P.g + rowi * kDK + 2 * lane), A.inv_tau);
                                qv[u] = *reinterpret_cast<const __half2 *>(P.q + rowi * kDK + 2 * lane);
                            }
                            acc.x += gv.x;
                            acc.y += gv.y;
                            pg[u] = acc;
                        }
                        *reinterpret_cast<float2 *>(htot + gw * 64 + 2 * lane) = acc;
                        named_sync(kBarG, kGThreads);
                        float2 offv = make_float2(0.f, 0.f);
                        for (int w = 0; w < gw; ++w) {
                            const float2 x = *reinterpret_cast<const float2 *>(htot + w * 64 + 2 * lane);
                            offv.x += x.x;
                            offv.y += x.y;
                        }
                        const float2 Dc = *reinterpret_cast<const float2 *>(dcum + ci * 64 + 2 * lane);
                        uint8_t *dst = sm + (qaddr[li] - sbase);
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const float2 qf = __half22float2(qv[u]);
                            sth2(dst + sw_off(t0 + u, 2 * lane),
                                 h2(qf.x * ex2a((offv.x + pg[u].x) * kLog2e) * Dc.x,
                                    qf.y * ex2a((offv.y + pg[u].y) * kLog2e) * Dc.y));
                        }
                        named_sync(kBarG, kGThreads);   // htot reused by the next chunk
                    }
                    (void)tg;
                }
                fence_proxy_async_cta();
                __syncthreads();
                if (warp == kWarpMMA) {
                    tc_fence_after();
                    if (elect_one_sync()) {
                        constexpr uint32_t id_o = idesc_f16_f32(64, kDV, false, true);
                        const uint32_t ba = sbase + L::sop;
                        for (int li = 0; li < nl; ++li)
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                umma_f16(tmem + 64 * li, desc_sw128(qaddr[li] + kk * 32, 16, 1024),
                                         desc_sw128(ba + kk * 2048, kTile, 1024), id_o, kk > 0 ? 1u : 0u);
                        umma_commit(bar(sm, B_FIX));
                    }
                    __syncwarp();
                }
                wait_l(bar(sm, B_FIX), n_fix & 1u, to);
                ++n_fix;
                tc_fence_after();
                // epilogues: teams RE (warps 6-9) and U (warps 2-5), chunk li on team li % 2
                if (warp >= kWarpU && warp < kWarpG) {
                    const int team = warp < kWarpRE ? 1 : 0;
                    const int q4 = warp & 3, tb = tid - (team ? kWarpU : kWarpRE) * 32;
                    int *rows = reinterpret_cast<int *>(sm + L::rowtab) + 64 * team;
                    for (int li = team; li < nl; li += 2) {
                        fill_rowtab(P, seq, c0 + list[li], rows, tb);
                        named_sync(team ? kBarT1 : kBarT0, 128);
                        uint32_t o[32];
                        ld_acc64(tmem + ((uint32_t)(32 * q4) << 16) + 64 * li, o);
                        tmem_ld_wait();
                        add_out_tile(P, o, q4, lane, rows);
                        named_sync(team ? kBarT1 : kBarT0, 128);
                    }
                }
                tc_fence_before();
                __syncthreads();
            }
        }
        __syncthreads();   // staging and state tiles are reused by the next sequence
    }

    // after a timeout some copy or MMA may still be in flight: give it time before
    // freeing tensor memory and leaving
    if (__syncthreads_or(to)) {
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 1000000ull) {
        }
    }
    if (warp == kWarpMMA) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace pp
}  // namespace gtr
