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
// Roles (one CTA = 16 warps, 128 registers each):
//   warps 0-3    state group U: S (fp32) lives in registers in the accumulator's
//                fragment layout; per chunk S <- d * (S + dS), and its fp16 copy is the
//                next chunk's S_prev operand.  Warp 0 owns the tensor memory and issues
//                the look-back's bulk copies of the earlier spans' aggregates;
//   warps 4-7    readout group RE: scores -> causal mask -> fp16 P back into tensor
//                memory; then the chunk's output tile -> fp16 -> coalesced row stores.
//                Warp 4 issues the tensor-core work (one elected lane): MMA 1 =
//                (K~^T V, Qint K~^T) and MMA 2 = Qint S_prev + P V, tcgen05 kind::f16
//                with fp32 accumulators in tensor memory, P read from tensor memory;
//   warps 8-15   gating group G, two teams of four warps, team t gating the chunks of
//                parity t: per chunk the cumulative decays, Qint and K~ (or the
//                sub-block operands, below) into 128-byte-swizzled operand tiles, and V
//                into its operand tile in scan order.  A team's first warp then loads
//                the chunk three ahead into the staging slot it freed: TMA tensor copies
//                of q, k, g, v into a 3-slot ring.  The scan direction is applied only in
//                the copies' coordinates: a chunk is a list of runs of grid tokens that
//                are contiguous in memory (a row segment, or a column segment at stride
//                W), each copied in memory order by boxes of 64, 32, .. 1 rows; the lanes
//                write the table staging row <- scan position (identity for L->R and
//                T->B, reversed inside each run for R->L and B->T).
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
constexpr int kPrefetchChunks = 8;           // chunks past the ring whose rows are prefetched for the corrections
constexpr int kThreads = 512;                // 16 warps (128 registers each)
constexpr int kWarpU = 0, kWarpRE = 4, kWarpG = 8;
constexpr int kUThreads = 128, kREThreads = 128, kGThreads = 256;
constexpr int kTeamThreads = 128;   // a gating team: 4 warps x 16 rows
// named barriers: gating teams 1 and 7 (team t: 1 + 6 t), all gating warps 8
constexpr uint32_t kBarU = 2, kBarRE = 3, kBarT0 = 5, kBarT1 = 6, kBarGAll = 8;
__host__ __device__ constexpr uint32_t bar_team(int team) { return 1u + 6u * (uint32_t)team; }
constexpr int kAggFloats = kDK * kDV + kDK;  // state + decay product
constexpr int kAggBytes = kAggFloats * 4;    // 16640
constexpr int kFoldSlots = 8;                // aggregates copied into smem at a time
constexpr int kFlagStride = 32;              // one 128-byte line per publish flag
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
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
    B_FULL = 0,     // [3][2] staging slot s landed, for a chunk of parity t (TMA transaction count)
    B_OPFULL = 6,   // [2] G done: Qint, K~, V, d, flags of a chunk
    B_MMA1 = 8,     // [2] MMA 1 complete
    B_SPFULL = 12,  // [2] S_prev operand written (U)
    B_MMA2 = 14,    // [2] MMA 2 complete (operands, S_prev, scores free; O ready)
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

// ------------------------------------------------------------------ staging loads
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
__device__ __noinline__ uint32_t issue_chunk(const Args &A, uint32_t slot, int seq, int cabs, uint32_t mbar,
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
#pragma unroll 1
            for (int lb = 6; lb >= 0; --lb) {
                if (!(len & (1 << lb))) continue;
                const uint32_t d = slot + (row0 + off) * 128u;
#pragma unroll 1
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

// Staging barrier of the CTA's chunk number gc: slot gc % 3, and one barrier per chunk
// parity, so that each barrier's phases belong to one gating team, which waits for them
// in order (a shared barrier could complete the other team's phase in between and
// alias the parity).
__device__ __forceinline__ uint32_t full_bar(uint32_t gc) { return B_FULL + 2u * (gc % kNStage) + (gc & 1u); }
__device__ __forceinline__ uint32_t full_parity(uint32_t gc) { return (gc / (2u * kNStage)) & 1u; }

// Chunk `cabs` of sequence `seq`, the CTA's chunk number gc, into its staging slot (one
// warp): the row table, the expected transaction bytes and the copies.
__device__ __noinline__ void load_chunk(const Args &A, uint8_t *sm, uint32_t sbase, uint32_t gc, int seq,
                                           int cabs, int lane) {
    const uint32_t s = gc % kNStage;
    write_meta(A.P, sm + L::meta + s * 128, cabs, lane);
    __syncwarp();
    if (lane == 0) {
        const uint32_t mb = smem_u32(bar(sm, full_bar(gc)));
        const uint32_t slot = sbase + L::stage + s * L::stage_bytes;
        mbar_arrive_expect_tx(bar(sm, full_bar(gc)), issue_chunk(A, slot, seq, cabs, mb, true));
        issue_chunk(A, slot, seq, cabs, mb, false);
    }
    __syncwarp();
}

// The first kNStage chunks of a sequence (chunk c goes to slot (gc0 + c) % kNStage: the
// sequence starts where the CTA's running chunk count stands, kept in the caller).
__device__ __forceinline__ void load_head(const Args &A, uint8_t *sm, uint32_t sbase, uint32_t gc0, int seq,
                                          int lane) {
    const int kspan = (int)blockIdx.x % A.PS;
    const int c0 = kspan * A.Lc;
    const int nch = min(A.Lc, A.P.n_chunks - c0);
    for (int c = 0; c < min(kNStage, nch); ++c) load_chunk(A, sm, sbase, gc0 + c, seq, c0 + c, lane);
}

// ------------------------------------------------------------------ gating (group G)
// Two gating teams of four warps; team b gates the chunks whose operands go to buffer b
// (every other chunk), so that two chunks are gated at once.  Warp w of a team owns the
// chunk's scan rows 16w .. 16w+15 (sub-block w of the sub-block path), lane l channels
// 2l, 2l+1.
struct GRegs {
    float2 p[16];   // prefix sums of the log-decay over a warp's 16 rows
};

// |x| of the eight fp16 values of a 16-byte word, as their bit patterns' per-half maximum
// (for non-negative fp16 values the bit patterns order like the values; a NaN orders
// above every finite value)
__device__ __forceinline__ uint32_t umax16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t absmax8(const uint4 &x) {
    return umax16x2(umax16x2(x.x & 0x7fff7fffu, x.y & 0x7fff7fffu), umax16x2(x.z & 0x7fff7fffu, x.w & 0x7fff7fffu));
}
__device__ __forceinline__ float half_bits_to_float(uint32_t h) {
    return __half2float(__ushort_as_half((unsigned short)h));
}

// Eight consecutive channels of a gate row as log-decays (from z when kZ).
template <bool kZ>
__device__ __forceinline__ void ld_gate8(const uint8_t *p, float (&g)[8], float inv_tau) {
    const uint4 w = *reinterpret_cast<const uint4 *>(p);
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&u[m]));
        g[2 * m] = f.x;
        g[2 * m + 1] = f.y;
    }
    if constexpr (kZ) {
#pragma unroll
        for (int j = 0; j < 8; ++j) g[j] = gate_of(g[j], inv_tau);
    }
}

__device__ __forceinline__ uint32_t hadd2_bits(uint32_t a, uint32_t b) {
    const __half2 r = __hadd2(*reinterpret_cast<const __half2 *>(&a), *reinterpret_cast<const __half2 *>(&b));
    return *reinterpret_cast<const uint32_t *>(&r);
}
__device__ __forceinline__ uint32_t hmul2_bits(uint32_t a, float x0, float x1) {
    const __half2 r = __hmul2(*reinterpret_cast<const __half2 *>(&a), h2(x0, x1));
    return *reinterpret_cast<const uint32_t *>(&r);
}

// Fast-path gating of the lane's four rows tb .. tb+3, channels 8 cg .. 8 cg + 7 (chunk
// decay >= e^-6, |k| <= 100): Qint = q exp(b), K~ = k exp(-b), with b (log2 units) the
// chunk-inclusive prefix sum x[i][j]; 16-byte loads and stores (a lane's eight channels
// are one 16-byte unit of the 128-byte-swizzled tile).  A held chunk also keeps Qint in
// its ring tile.  (Two instances: a branch inside the unrolled loop would keep the
// scheduler from overlapping the rows.)
template <bool kHeld>
__device__ __forceinline__ void gate_fast(const float (&x)[4][8], const uint8_t *st, uint32_t rw, int tb, int nrows,
                                          int cg, uint8_t *qo, uint8_t *ko, uint8_t *ro) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int t = tb + i;
        const uint32_t o = ((rw >> (8 * i)) & 0xffu) * 128u + 16u * (uint32_t)cg;
        const bool ok = t < nrows;
        uint4 q4 = *reinterpret_cast<const uint4 *>(st + L::st_q + o);
        uint4 k4 = *reinterpret_cast<const uint4 *>(st + L::st_k + o);
        if (!ok) q4 = k4 = make_uint4(0u, 0u, 0u, 0u);   // rows past the grid
        uint4 qi, ki;
        qi.x = hmul2_bits(q4.x, ex2a(x[i][0]), ex2a(x[i][1]));
        qi.y = hmul2_bits(q4.y, ex2a(x[i][2]), ex2a(x[i][3]));
        qi.z = hmul2_bits(q4.z, ex2a(x[i][4]), ex2a(x[i][5]));
        qi.w = hmul2_bits(q4.w, ex2a(x[i][6]), ex2a(x[i][7]));
        ki.x = hmul2_bits(k4.x, ex2a(-x[i][0]), ex2a(-x[i][1]));
        ki.y = hmul2_bits(k4.y, ex2a(-x[i][2]), ex2a(-x[i][3]));
        ki.z = hmul2_bits(k4.z, ex2a(-x[i][4]), ex2a(-x[i][5]));
        ki.w = hmul2_bits(k4.w, ex2a(-x[i][6]), ex2a(-x[i][7]));
        const uint32_t so = (uint32_t)t * 128u + ((uint32_t)(cg ^ (t & 7)) << 4);
        *reinterpret_cast<uint4 *>(qo + so) = qi;
        *reinterpret_cast<uint4 *>(ko + so) = ki;
        if constexpr (kHeld) *reinterpret_cast<uint4 *>(ro + so) = qi;
    }
}

// Exact fp32 diagonal blocks of the flagged sub-blocks (rare: decay below e^-8 inside 16
// tokens, or keys too large): value(u, w) = sum_i q[u] k[w] exp(sum_{r=w+1..u} g[r]),
// stored as fp16 (it becomes an fp16 P entry anyway).  The team's 128 threads.
template <bool kZ>
__device__ __noinline__ void exact_diag(const uint8_t *st, const uint8_t *meta, int nrows, const int *flags,
                                        __half *dst, int tt, float inv_tau) {
    for (int task = tt; task < 4 * 256; task += kTeamThreads) {
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
// registers).  Warp gw's rows are sub-block I = gw, ht[J] the total log-decay of block J.
// Writes Qint and K^ = K * exp(b_C - b) into qo / ko (and Qint into ro when held), flags
// the diagonal blocks that need the exact evaluation, evaluates those into diagx[b], then
// overlays Qd, Kd, A_J and B_J on the chunk's staging slot.
template <bool kZ>
__device__ __noinline__ void gate_slow(uint8_t *sm, const float *htot, int gw, int lane, int tt, uint32_t bid,
                                       uint8_t *st, const uint8_t *meta, int nrows, uint8_t *qo, uint8_t *ko,
                                       uint8_t *ro, bool held, int *bfl, int b, float inv_tau) {
    const int t0 = 16 * gw, I = gw;
    // the team's block totals (kept in log2 units) in natural-log units, for the lane's
    // channels 2 lane, 2 lane + 1
    float2 ht[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const float2 h = *reinterpret_cast<const float2 *>(htot + w * 64 + 2 * lane);
        ht[w] = make_float2(h.x * kLn2, h.y * kLn2);
    }
    if (tt < 4) bfl[tt] = 0;   // (the readout of this buffer's previous chunk is complete)
    named_sync(bid, kTeamThreads);
    __half2 qh[16], kh[16];
    float2 gr[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
        const bool ok = t0 + u < nrows;
        const uint32_t so = (uint32_t)meta[t0 + u] * 128u + 4u * (uint32_t)lane;
        const uint32_t qb = *reinterpret_cast<const uint32_t *>(st + L::st_q + so);
        const uint32_t kb = *reinterpret_cast<const uint32_t *>(st + L::st_k + so);
        const uint32_t qz = ok ? qb : 0u, kz = ok ? kb : 0u;
        qh[u] = *reinterpret_cast<const __half2 *>(&qz);
        kh[u] = *reinterpret_cast<const __half2 *>(&kz);
        const float2 gv = ld_gate2<kZ>(st + L::st_g + so, inv_tau);
        gr[u] = ok ? gv : make_float2(0.f, 0.f);
    }
    GRegs R;   // inclusive prefix sums within the warp's block
    {
        float2 a = make_float2(0.f, 0.f);
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            a.x += gr[u].x;
            a.y += gr[u].y;
            R.p[u] = a;
        }
    }
    float2 pre = make_float2(0.f, 0.f), post = make_float2(0.f, 0.f);
#pragma unroll
    for (int J = 0; J < 4; ++J) {
        if (J < I) { pre.x += ht[J].x; pre.y += ht[J].y; }
        if (J > I) { post.x += ht[J].x; post.y += ht[J].y; }
    }
    float2 bs[16];   // within-block suffix sums (excluding the row)
    {
        float2 a = make_float2(0.f, 0.f);
#pragma unroll
        for (int u = 15; u >= 0; --u) {
            bs[u] = a;
            a.x += gr[u].x;
            a.y += gr[u].y;
        }
    }
    bool kbad = !(ht[I].x >= kDiagMinLogTotal) || !(ht[I].y >= kDiagMinLogTotal);
#pragma unroll
    for (int u = 0; u < 16; ++u) {
        const float2 bp = R.p[u];
        const float2 qf = __half22float2(qh[u]), kf = __half22float2(kh[u]);
        const __half2 qi = h2(qf.x * ex2a((pre.x + bp.x) * kLog2e), qf.y * ex2a((pre.y + bp.y) * kLog2e));
        const uint32_t o = sw_off(t0 + u, 2 * lane);
        sth2(qo + o, qi);
        sth2(ko + o, h2(kf.x * ex2a((bs[u].x + post.x) * kLog2e), kf.y * ex2a((bs[u].y + post.y) * kLog2e)));
        if (held) sth2(ro + o, qi);
        const float kd0 = kf.x * ex2a(-bp.x * kLog2e), kd1 = kf.y * ex2a(-bp.y * kLog2e);
        kbad |= !(fabsf(kd0) <= kDiagMaxK) || !(fabsf(kd1) <= kDiagMaxK);
    }
    if (__any_sync(0xffffffffu, kbad) && lane == 0) atomicOr(&bfl[I], 1);
    named_sync(bid, kTeamThreads);
    const bool anyflag = (bfl[0] | bfl[1] | bfl[2] | bfl[3]) != 0;
    if (anyflag)
        exact_diag<kZ>(st, meta, nrows, bfl, reinterpret_cast<__half *>(sm + L::diagx + b * 2048), tt, inv_tau);
    named_sync(bid, kTeamThreads);   // raw rows no longer read: overlay the operands
    const bool fl = bfl[I] != 0;
#pragma unroll
    for (int u = 0; u < 16; ++u) {
        const int t = t0 + u;
        const float2 bp = R.p[u];
        const float2 qf = __half22float2(qh[u]), kf = __half22float2(kh[u]);
        sth2(st + L::sl_qa + sw_off(t, 2 * lane),
             h2(qf.x * ex2a(bp.x * kLog2e), qf.y * ex2a(bp.y * kLog2e)));
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
                acc.x += ht[J].x;   // one more block between row and anchor
                acc.y += ht[J].y;
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
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x8.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}
// Columns 64..111 of a scores buffer (the blocks below the diagonal), the same register
// order as ld_acc64 for columns 0..47; registers 24..31 stay zero.
__device__ __forceinline__ void ld_off48(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x4.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.ld.sync.aligned.16x256b.x2.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
                   "=r"(r[23])
                 : "r"(taddr + 32)
                 : "memory");
#pragma unroll
    for (int e = 24; e < 32; ++e) r[e] = 0u;
}

// Output tile (fp32 in registers, fragment layout) -> fp16 -> staging -> coalesced rows.
// Team of 4 warps (128 threads, named barrier `bid`); returns the thread's max |o|.
// The chunk's output tile: fp16 through the staging tile `os`, then 16-byte row pieces
// to the token rows (`rows`; -1: past the grid).  With P.acc (the second key-channel
// half of a dk = 128 call) each piece is added to what the first half stored (a plain
// read-modify-write: the launches are ordered on the stream).  Returns max |value|
// written, for the range check (the sum, when adding).
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
    if (!P.acc) {
#pragma unroll
        for (int x = tb; x < 64 * 8; x += 128) {
            const int row = x >> 3, c8 = x & 7;
            const int ro = rows[row];
            if (ro >= 0)
                *reinterpret_cast<uint4 *>(P.out + (size_t)ro * P.ldv + 8 * c8) =
                    *reinterpret_cast<const uint4 *>(os + sw_off(row, 8 * c8));
        }
    } else {
        uint4 cur[4];
        int ro[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {   // the loads first, so that their latencies overlap
            const int x = tb + 128 * i, row = x >> 3, c8 = x & 7;
            ro[i] = rows[row];
            cur[i] = *reinterpret_cast<const uint4 *>(P.out + (size_t)(ro[i] >= 0 ? ro[i] : 0) * P.ldv + 8 * c8);
        }
        __half2 m2 = __float2half2_rn(0.f);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int x = tb + 128 * i, row = x >> 3, c8 = x & 7;
            const uint4 a = *reinterpret_cast<const uint4 *>(os + sw_off(row, 8 * c8));
            uint4 v;
            v.x = hadd2_bits(cur[i].x, a.x);
            v.y = hadd2_bits(cur[i].y, a.y);
            v.z = hadd2_bits(cur[i].z, a.z);
            v.w = hadd2_bits(cur[i].w, a.w);
            if (ro[i] >= 0) {
                *reinterpret_cast<uint4 *>(P.out + (size_t)ro[i] * P.ldv + 8 * c8) = v;
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int m = 0; m < 4; ++m) m2 = __hmax2_nan(m2, __habs2(*reinterpret_cast<const __half2 *>(&w4[m])));
            }
        }
        // the sum is what must stay inside fp16 (an overflow shows as inf, a NaN stays NaN)
        const float ml = __low2float(m2), mh = __high2float(m2);
        mx = (ml != ml || mh != mh) ? ml + mh : fmaxf(mx, fmaxf(ml, mh));
    }
    named_sync(bid, 128);
    return mx;
}

// Correction tile (fp32, fragment layout) added onto the stored fp16 outputs with
// reductions (one addend per element: the result does not depend on their order).
// Adds a 64x64 fp32 fragment tile (the correction term) to output rows this CTA has
// already stored: a plain read-modify-write (no other CTA writes these rows, and the
// CTA's barriers since the store make it visible), staged through `os` so that every
// access is a 16-byte row piece; the correction is rounded to fp16 before the add.
__device__ __forceinline__ void add_out_tile(const Params &P, const uint32_t (&r)[32], int q4, int lane, int tb,
                                             uint8_t *os, const int *rows, uint32_t bid) {
    const int r0 = 16 * q4 + (lane >> 2), a2 = 2 * (lane & 3);
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
        const int h = e >> 4, j = (e >> 2) & 3, hh = (e >> 1) & 1;
        sth2(os + sw_off(r0 + 8 * hh, 32 * h + 8 * j + a2), h2(__uint_as_float(r[e]), __uint_as_float(r[e + 1])));
    }
    named_sync(bid, 128);
    uint4 cur[4], add[4];
    int ro[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {   // the loads first, so that their latencies overlap
        const int x = tb + 128 * i, row = x >> 3, c8 = x & 7;
        ro[i] = rows[row];
        const int rr = ro[i] >= 0 ? ro[i] : 0;
        cur[i] = *reinterpret_cast<const uint4 *>(P.out + (size_t)rr * P.ldv + 8 * c8);
        add[i] = *reinterpret_cast<const uint4 *>(os + sw_off(row, 8 * c8));
    }
    __half2 m2 = __float2half2_rn(0.f);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int x = tb + 128 * i, c8 = x & 7;
        if (ro[i] >= 0) {
            uint4 v;
            v.x = hadd2_bits(cur[i].x, add[i].x);
            v.y = hadd2_bits(cur[i].y, add[i].y);
            v.z = hadd2_bits(cur[i].z, add[i].z);
            v.w = hadd2_bits(cur[i].w, add[i].w);
            *reinterpret_cast<uint4 *>(P.out + (size_t)ro[i] * P.ldv + 8 * c8) = v;
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int m = 0; m < 4; ++m) m2 = __hmax2_nan(m2, __habs2(*reinterpret_cast<const __half2 *>(&w4[m])));
        }
    }
    const float ml = __low2float(m2), mh = __high2float(m2);
    range_check(ml != ml || mh != mh ? ml + mh : fmaxf(ml, mh));   // the corrected outputs
    named_sync(bid, 128);
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

// Scores of a sub-block-path chunk -> causal fp16 P (out of line: rare).  Rows of this
// warp's quarter q4 are sub-block q4; a column in key block J < q4 takes the block below
// the diagonal (columns 64..111 of the scores buffer), J == q4 the diagonal block (or its
// exact evaluation), J > q4 zero.  Returns the largest |P|.
__device__ __noinline__ float readout_slow(uint8_t *sm, uint32_t ta, const uint32_t (&sc)[32], uint32_t (&pv)[16],
                                           uint32_t b, int q4, int r0, int a2) {
    uint32_t of[32];   // (key block 3 is never below the diagonal)
    ld_off48(ta + 64, of);
    tmem_ld_wait();
    const int *fl = reinterpret_cast<const int *>(sm + L::bflag) + 4 * b;
    const bool exact = fl[q4] != 0;
    const __half *dx = reinterpret_cast<const __half *>(sm + L::diagx + b * 2048) + q4 * 256;
    float pmx = 0.f;
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
    return pmx;
}

// Phase-4 B operand of held chunk i (D_i * S_in): free operand tiles after the pipeline.
__host__ __device__ constexpr int held_tile(int i) { return i == 0 ? L::sop : i == 1 ? L::sop + kTile : L::vop; }
static_assert(kRing == 3, "three held tiles");

// ------------------------------------------------------------------ MMA issue
// MMA 1 of the chunk in operand buffer b (staging slot s): dS = K~^T V (K^ on the
// sub-block path) and the scores Qint K~^T, or the diagonal and below-diagonal sub-block
// products.  Called by a converged warp; one elected lane issues and commits.
// Descriptors of the k-steps of one operand differ only in the start-address field
// (bits 0..13, address / 16): shared memory addresses stay below 2^18, so adding the
// step's byte offset / 16 to a base descriptor never carries out of the field.
__device__ __forceinline__ uint64_t desc_step(uint64_t d, uint32_t bytes) { return d + (bytes >> 4); }

__device__ __forceinline__ void issue_mma1(uint8_t *sm, uint32_t sbase, uint32_t tmem, uint32_t b, uint32_t s,
                                           bool slow) {
    constexpr uint32_t id_ds = idesc_f16_f32(64, kDV, true, true);
    constexpr uint32_t id_sc = idesc_f16_f32(64, 64, false, false);
    constexpr uint32_t id_off = idesc_f16_f32(64, 16, false, false);
    const uint32_t kta = sbase + L::kt + b * kTile, va = sbase + L::vop + b * kTile;
    const uint32_t qa = sbase + L::qint + b * kTile;
    const uint32_t sl = sbase + L::stage + s * L::stage_bytes;
    const uint32_t dsc = tmem + kColDS + 64 * b, scc = tmem + kColScores + 128 * b;
    if (elect_one_sync()) {
        const uint64_t dk_mn = desc_sw128(kta, kTile, 1024), dv_mn = desc_sw128(va, kTile, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            umma_f16(dsc, desc_step(dk_mn, kk * 2048), desc_step(dv_mn, kk * 2048), id_ds, kk > 0 ? 1u : 0u);
        if (!slow) {
            const uint64_t dq = desc_sw128(qa, 16, 1024), dk = desc_sw128(kta, 16, 1024);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                umma_f16(scc, desc_step(dq, kk * 32), desc_step(dk, kk * 32), id_sc, kk > 0 ? 1u : 0u);
        } else {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                umma_f16(scc, desc_sw128(sl + L::sl_qa + kk * 32, 16, 1024),
                         desc_sw128(sl + L::sl_kd + kk * 32, 16, 1024), id_sc, kk > 0 ? 1u : 0u);
            // A_J's descriptor starts 16(J+1) rows before its region, so that row t of the
            // operand is scan row t (earlier rows: finite values of the regions before it,
            // whose results are never read)
#pragma unroll
            for (int J = 0; J < 3; ++J) {
                const uint32_t abase = J == 0 ? 48u * 128u : J == 1 ? 80u * 128u : 96u * 128u;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_f16(scc + 64 + 16 * J, desc_sw128(sl + L::sl_qa + abase + kk * 32, 16, 1024),
                             desc_sw128(sl + L::sl_b + J * 2048 + kk * 32, 16, 1024), id_off, kk > 0 ? 1u : 0u);
            }
        }
        umma_commit(bar(sm, B_MMA1 + b));
    }
    __syncwarp();
}

// MMA 2 of the chunk in operand buffer b: O = Qint S_prev + P V, P read from the scores'
// tensor memory.  `last`: also signals the drain barrier (every MMA of the sequence).
__device__ __forceinline__ void issue_mma2(uint8_t *sm, uint32_t sbase, uint32_t tmem, uint32_t b, bool last) {
    constexpr uint32_t id_o = idesc_f16_f32(64, kDV, false, true);
    const uint32_t qa = sbase + L::qint + b * kTile, sa = sbase + L::sop + b * kTile;
    const uint32_t va = sbase + L::vop + b * kTile;
    const uint32_t oc = tmem + kColO + 64 * b, pc = tmem + kColScores + 128 * b;
    if (elect_one_sync()) {
        const uint64_t dq = desc_sw128(qa, 16, 1024), ds = desc_sw128(sa, kTile, 1024);
        const uint64_t dv = desc_sw128(va, kTile, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            umma_f16(oc, desc_step(dq, kk * 32), desc_step(ds, kk * 2048), id_o, kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)   // P from TMEM: K step 16 = 8 packed columns
            umma_f16_ta(oc, pc + 8 * kk, desc_step(dv, kk * 2048), id_o, 1u);
        umma_commit(bar(sm, B_MMA2 + b));
        if (last) umma_commit(bar(sm, B_DRAIN));
    }
    __syncwarp();
}

// ------------------------------------------------------------------ kernel
// kZ: the third input holds the gate pre-activation z instead of the log-decay g.
template <bool kZ>
__global__ void __launch_bounds__(kThreads, 1) gla_fwd_pipe_kernel(const __grid_constant__ Args A) {
    extern __shared__ uint8_t smem_raw[];
    // aligned by an offset from the shared array itself (not through an integer), so
    // that the compiler still sees every tile access as shared memory
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(sm);
    const Params &P = A.P;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int PS = A.PS;
    const int kspan = (int)blockIdx.x % PS;
    const int grp = (int)blockIdx.x / PS, ngrp = (int)gridDim.x / PS;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + L::tslot);
    float *dcum = reinterpret_cast<float *>(sm + L::dcum);
    float *cmeta = reinterpret_cast<float *>(sm + L::cmeta);

    if (warp == kWarpU) {
        tmem_alloc(tslot, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < 2 * kNStage; ++i) mbar_init(bar(sm, B_FULL + i), 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(sm, B_OPFULL + i), 1);
            mbar_init(bar(sm, B_MMA1 + i), 1);
            mbar_init(bar(sm, B_SPFULL + i), 1);
            mbar_init(bar(sm, B_MMA2 + i), 1);
        }
        mbar_init(bar(sm, B_AGG), 1);
        mbar_init(bar(sm, B_FIX), 1);
        mbar_init(bar(sm, B_DRAIN), 1);
        fence_mbar_init();
    }
    if (warp == kWarpG && lane < 28 && (lane & 7) < 7 && ((A.used >> (lane & 7)) & 1u))
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&A.maps.m[lane >> 3][lane & 7]))
                     : "memory");
    // the first chunk's rows into L2 while the grid ahead drains (L2 is where every
    // SM's accesses meet, so a later write by that grid still reaches the copies)
    if (warp == kWarpG && lane == 0 && grp < P.n_seq && P.dir == GTR_L2R) {
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
    if (warp == kWarpG && grp < P.n_seq) load_head(A, sm, sbase, 0u, grp, lane);
    uint32_t n_agg = 0, n_fix = 0, n_drain = 0;

    for (int seq = grp; seq < P.n_seq; seq += ngrp) {
        const int c0 = kspan * A.Lc;
        const int nch = min(A.Lc, P.n_chunks - c0);   // >= 1 (host guarantees)
        const bool later = kspan > 0;
        const bool publish = PS > 1 && kspan < PS - 1;
        const int nring = later ? min(kRing, nch) : 0;

        if (warp < kWarpRE) {
            // ======================================================= state group U
            const int q4 = warp & 3, ut = tid - kWarpU * 32;
            const int r0 = 16 * q4 + (lane >> 2);
            float S[32];
            {
                const float *s0 = (!later && P.s0 != nullptr) ? P.s0 + (size_t)seq * P.sstride : nullptr;
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const int h = e >> 4, j = (e >> 2) & 3, hh = (e >> 1) & 1;
                    float2 v = make_float2(0.f, 0.f);
                    if (s0) v = *reinterpret_cast<const float2 *>(s0 + (r0 + 8 * hh) * P.ldv + 32 * h + 8 * j + 2 * (lane & 3));
                    S[e] = v.x;
                    S[e + 1] = v.y;
                }
            }
            // S_prev of the first chunk; then (for the next chunk's d and flags, and so
            // that G cannot complete that buffer's next phase before this wait) G's signal
            float dn0, dn1;
            bool slown;
            // decay products from the span start for rows r0, r0+8 (D_c of chunk c), kept
            // for the held chunks and the publish, and recorded in dcum for phase 4
            float D0 = 1.f, D1 = 1.f;
            float Dh0[kRing], Dh1[kRing];
#pragma unroll
            for (int i = 0; i < kRing; ++i) Dh0[i] = Dh1[i] = 1.f;
            if ((lane & 3) == 0) {
                dcum[r0] = 1.f;
                dcum[r0 + 8] = 1.f;
            }
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
                if (warp == kWarpU) {
                    tc_fence_after();
                    issue_mma1(sm, sbase, tmem, bn, gn % kNStage, slown);
                }
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
                tmem_ld_wait();   // (warp-collective: every lane's loads are complete)
                // MMA 1 of chunk c+1, if its operands are ready already.  Its dS block held
                // dS of chunk c-1, read by every warp of the group before the group's barrier
                // of the previous iteration; its scores block P of chunk c-1, read by MMA 2
                // of chunk c-1, which G waited for before gating chunk c+1.
                bool issued = false;
                if (warp == kWarpU && c + 1 < nch) {
                    const uint32_t gn = gc + 1, bn = gn & 1u;
                    if (mbar_test(bar(sm, B_OPFULL + bn), (gn >> 1) & 1u)) {
                        tc_fence_after();
                        issue_mma1(sm, sbase, tmem, bn, gn % kNStage,
                                   reinterpret_cast<const int *>(sm + L::slowf)[bn] != 0);
                        issued = true;
                    }
                }
                tc_fence_before();
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const float d = ((e >> 1) & 1) ? d1 : d0;
                    const float x = __uint_as_float(ds[e]);
                    S[e] = slow ? fmaf(d, S[e], x) : d * (S[e] + x);
                }
                D0 *= d0;
                D1 *= d1;
#pragma unroll
                for (int i = 1; i < kRing; ++i)
                    if (c + 1 == i) {
                        Dh0[i] = D0;
                        Dh1[i] = D1;
                    }
                if ((lane & 3) == 0 && c + 1 <= kMaxSpan) {
                    dcum[(c + 1) * 64 + r0] = D0;
                    dcum[(c + 1) * 64 + r0 + 8] = D1;
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
                    if (warp == kWarpU && !issued) {
                        tc_fence_after();
                        issue_mma1(sm, sbase, tmem, bn, gn % kNStage, slown);
                    }
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
                named_sync(kBarU, kUThreads);   // dcum[nch]: one writer per row
                if (ut < 64) agg[kDK * kDV + ut] = dcum[nch * 64 + ut];
                named_sync(kBarU, kUThreads);
                if (ut == 0)   // readers to come: spans kspan+1 .. PS-1
                    sp::st_release_gpu(A.flags + ((size_t)seq * PS + kspan) * kFlagStride, (unsigned)(PS - 1 - kspan));
            }
            if (PS == 1 && P.sf != nullptr) {
                float *sf = P.sf + (size_t)seq * P.sstride;
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const int h = e >> 4, j = (e >> 2) & 3, hh = (e >> 1) & 1;
                    *reinterpret_cast<float2 *>(sf + (r0 + 8 * hh) * P.ldv + 32 * h + 8 * j + 2 * (lane & 3)) =
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
            // every MMA of this sequence's chunks complete: the operand tiles that the
            // look-back slots overlay are free (a dedicated barrier with one phase per
            // sequence, so that no parity wait can match an earlier phase)
            wait_l(bar(sm, B_DRAIN), n_drain & 1u, to);
            ++n_drain;
            if (later) {
                // ---------------- phase 3: look back over spans 0 .. kspan-1
                float Sin[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) Sin[e] = 0.f;
                for (int j0 = 0; j0 < kspan; j0 += kFoldSlots) {
                    const int nj = min(kFoldSlots, kspan - j0);
                    if (warp == kWarpU) {
                        // lane u polls span j0+u's flag and copies that aggregate at once (the
                        // slots overlay the staging ring and the first operand tiles, free once
                        // the drain barrier has completed)
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
                    }
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
                    named_sync(kBarU, kUThreads);   // slots free for the next batch
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
                // S_in as the fp16 B operands of the correction MMAs: D_c * S_in (rows
                // scaled) for the held chunks c (their ring tiles hold Qint), S_in itself for
                // the rebuilt ones (Qint * D_c rebuilt)
                range_check(fmaxf(m0, m1));
                write_state_tile(sm + L::vop + kTile, Sin, q4, lane);
#pragma unroll
                for (int i = 0; i < kRing; ++i) {
                    if (i >= nring) break;
                    float Ss[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) Ss[e] = Sin[e] * (((e >> 1) & 1) ? Dh1[i] : Dh0[i]);
                    write_state_tile(sm + held_tile(i), Ss, q4, lane);
                }
                if (kspan == PS - 1 && P.sf != nullptr) {   // final state D_span * S_in + S_local
                    const float G0 = D0, G1 = D1;
                    float *sf = P.sf + (size_t)seq * P.sstride;
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const int h = e >> 4, j = (e >> 2) & 3, hh = (e >> 1) & 1;
                        const float Gd = hh ? G1 : G0;
                        const float4 pk = park[(e >> 2) * 128 + q4 * 32 + lane];   // S_local[4m .. 4m+3]
                        const float sx = (e & 2) ? pk.z : pk.x, sy = (e & 2) ? pk.w : pk.y;
                        *reinterpret_cast<float2 *>(sf + (r0 + 8 * hh) * P.ldv + 32 * h + 8 * j + 2 * (lane & 3)) =
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
                        // copies for the out-of-line call: sc and pv never have their address
                        // taken, so that the fast path keeps them in registers
                        uint32_t scs[32], pvs[16];
                        tmem_ld_wait();   // (the scores' loads complete before they are copied)
#pragma unroll
                        for (int e = 0; e < 32; ++e) scs[e] = sc[e];
                        pmx = readout_slow(sm, ta, scs, pvs, b, q4, r0, a2);
#pragma unroll
                        for (int e = 0; e < 16; ++e) pv[e] = pvs[e];
                    }
                    range_check(pmx);
                    tmem_st_16x128b_x8(ta, pv);
                    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                    tc_fence_before();
                    named_sync(kBarRE, kREThreads);   // P complete; O of chunk c-2 read by every RE warp
                    if (warp == kWarpRE) {
                        // MMA 2 of chunk c, once U has written its S_prev
                        wait_l(bar(sm, B_SPFULL + b), ph, to);
                        tc_fence_after();
                        issue_mma2(sm, sbase, tmem, b, c + 1 == nch);
                    }
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
            // team b gates the chunks whose global index has parity b (operand buffer b)
            const int team = (warp - kWarpG) >> 2, gw = (warp - kWarpG) & 3;
            const int tt = tid - (kWarpG + 4 * team) * 32, t0 = 16 * gw;
            const uint32_t bid = bar_team(team);
            float *htot = reinterpret_cast<float *>(sm + L::htot) + team * 4 * 64;
            // lane layout: row slot rs = lane / 8 (rows tb .. tb+3 of the warp's 16),
            // channel group cg = lane % 8 (channels 8 cg .. 8 cg + 7: one 16-byte unit)
            const int cg = lane & 7, rs = lane >> 3, tb = t0 + 4 * rs;
            for (int c = (int)(((uint32_t)team - gc0) & 1u); c < nch; c += 2) {
                const uint32_t gc = gc0 + c, b = gc & 1u, s = gc % kNStage, ph = (gc >> 1) & 1u;
                const bool held = c < nring;
                wait_l(bar(sm, full_bar(gc)), full_parity(gc), to);
                uint8_t *st = sm + L::stage + s * L::stage_bytes;
                const uint8_t *meta = sm + L::meta + s * 128;
                const int nrows = *reinterpret_cast<const int *>(meta + 64);
                unsigned *wm = reinterpret_cast<unsigned *>(sm + L::wmax) + 16 * team;
                // ---------- pass 1: prefix sums of the log-decay (log2 units) over the
                // lane's rows, then over the warp's row slots; maxima of |q| and |k|
                const uint32_t rw = *reinterpret_cast<const uint32_t *>(meta + tb);   // staging rows
                float x[4][8];
                {
                    float acc[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) acc[j] = 0.f;
                    uint32_t qm = 0u, km = 0u;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint32_t o = ((rw >> (8 * i)) & 0xffu) * 128u + 16u * (uint32_t)cg;
                        const bool ok = tb + i < nrows;   // rows past the grid count as zero
                        float gv[8];
                        ld_gate8<kZ>(st + L::st_g + o, gv, A.inv_tau);
                        const uint32_t qa = absmax8(*reinterpret_cast<const uint4 *>(st + L::st_q + o));
                        const uint32_t ka = absmax8(*reinterpret_cast<const uint4 *>(st + L::st_k + o));
                        qm = ok ? umax16x2(qm, qa) : qm;
                        km = ok ? umax16x2(km, ka) : km;
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            acc[j] = ok ? fmaf(gv[j], kLog2e, acc[j]) : acc[j];
                            x[i][j] = acc[j];
                        }
                    }
                    float tot[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {   // inclusive scan over the row slots
                        float v = acc[j];
                        float y = __shfl_up_sync(0xffffffffu, v, 8);
                        v += rs >= 1 ? y : 0.f;
                        y = __shfl_up_sync(0xffffffffu, v, 16);
                        v += rs >= 2 ? y : 0.f;
                        tot[j] = v;
                        const float ex = v - acc[j];   // the warp's rows before the lane's
#pragma unroll
                        for (int i = 0; i < 4; ++i) x[i][j] += ex;
                    }
                    if (rs == 3) {   // the warp's block totals
                        float4 *hp = reinterpret_cast<float4 *>(htot + gw * 64 + 8 * cg);
                        hp[0] = make_float4(tot[0], tot[1], tot[2], tot[3]);
                        hp[1] = make_float4(tot[4], tot[5], tot[6], tot[7]);
                    }
                    const unsigned wq = __reduce_max_sync(0xffffffffu, max(qm & 0xffffu, qm >> 16));
                    const unsigned wk = __reduce_max_sync(0xffffffffu, max(km & 0xffffu, km >> 16));
                    if (lane == 0) {
                        wm[gw] = wq;
                        wm[4 + gw] = wk;
                    }
                }
                named_sync(bid, kTeamThreads);
                // ---------- pass 2
                float bC[8];
                {
                    float off[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) off[j] = bC[j] = 0.f;
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const float4 *hp = reinterpret_cast<const float4 *>(htot + w * 64 + 8 * cg);
                        const float4 h0 = hp[0], h1 = hp[1];
                        const float hv[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            bC[j] += hv[j];
                            off[j] += w < gw ? hv[j] : 0.f;
                        }
                    }
#pragma unroll
                    for (int i = 0; i < 4; ++i)
#pragma unroll
                        for (int j = 0; j < 8; ++j) x[i][j] += off[j];
                }
                const uint4 wq4 = *reinterpret_cast<const uint4 *>(wm), wk4 = *reinterpret_cast<const uint4 *>(wm + 4);
                const float qmx = half_bits_to_float(max(max(wq4.x, wq4.y), max(wq4.z, wq4.w)));
                const float kmx = half_bits_to_float(max(max(wk4.x, wk4.y), max(wk4.z, wk4.w)));
                bool bad = !(kmx <= kFastMaxK);
#pragma unroll
                for (int j = 0; j < 8; ++j) bad |= !(bC[j] >= kFastMinLogDecay * kLog2e);
                // every warp's lanes cover all 64 channels: a warp vote is the chunk's decision
                const bool slow = __any_sync(0xffffffffu, bad);
                // operand buffers b free (MMA 2 of chunk gc-2 complete)
                if (gc >= 2) wait_l(bar(sm, B_MMA2 + b), ph ^ 1u, to);
                // V rows into the scan-ordered operand tile (row tt/2, 16-byte units
                // 4 (tt%2) .. +3)
                {
                    const int t = tt >> 1, pc = 4 * (tt & 1);
                    const int r = meta[t];
                    const uint8_t *vs = st + L::st_v + r * 128 + 16 * pc;
                    uint4 v[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) v[i] = *reinterpret_cast<const uint4 *>(vs + 16 * i);
                    uint8_t *vo = sm + L::vop + b * kTile;
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        *reinterpret_cast<uint4 *>(vo + sw_off(t, 8 * (pc + i))) =
                            t < nrows ? v[i] : make_uint4(0u, 0u, 0u, 0u);
                }
                uint8_t *qo = sm + L::qint + b * kTile;
                uint8_t *ko = sm + L::kt + b * kTile;
                uint8_t *ro = sm + L::ring + (held ? c : 0) * kTile;
                int *bfl = reinterpret_cast<int *>(sm + L::bflag) + 4 * b;
                if (!slow) {
                    if (held)
                        gate_fast<true>(x, st, rw, tb, nrows, cg, qo, ko, ro);
                    else
                        gate_fast<false>(x, st, rw, tb, nrows, cg, qo, ko, ro);
                } else {
                    gate_slow<kZ>(sm, htot, gw, lane, tt, bid, st, meta, nrows, qo, ko, ro, held, bfl, b, A.inv_tau);
                }
                // the chunk's decay (the state group keeps the products from the span start)
                if (gw == 0 && rs == 0) {
                    float4 *dp = reinterpret_cast<float4 *>(sm + L::dloc + b * 256 + 32 * cg);
                    dp[0] = make_float4(ex2a(bC[0]), ex2a(bC[1]), ex2a(bC[2]), ex2a(bC[3]));
                    dp[1] = make_float4(ex2a(bC[4]), ex2a(bC[5]), ex2a(bC[6]), ex2a(bC[7]));
                    if (lane == 0 && c < kMaxSpan) cmeta[2 * c] = qmx;
                }
                fence_proxy_async_cta();
                named_sync(bid, kTeamThreads);
                if (tt == 0) {
                    reinterpret_cast<int *>(sm + L::slowf)[b] = slow ? 1 : 0;
                    mbar_arrive(bar(sm, B_OPFULL + b));   // MMA 1 may be issued
                }
                // the slot is free: the team's first warp loads chunk c+3 into it (on the
                // sub-block path MMA 1 reads operands overlaid on the slot: after it completes)
                if (gw == 0 && c + kNStage < nch) {
                    if (slow) wait_l(bar(sm, B_MMA1 + b), ph, to);
                    load_chunk(A, sm, sbase, gc + kNStage, seq, c0 + c + kNStage, lane);
                }
            }
            if (later) {
                // while the state group looks back: the q and g rows of the chunks past
                // the ring (the ones the corrections may rebuild) into L2
                const int bb = seq / P.heads, hh = seq - bb * P.heads;
                const int gt = tid - kWarpG * 32;
                const int npf = min(nch, kRing + kPrefetchChunks) - kRing;
                for (int i = gt; i < npf * 2 * kChunk; i += kGThreads) {
                    const int ci = kRing + i / (2 * kChunk), t = (i >> 1) & (kChunk - 1);
                    const int p = (c0 + ci) * kChunk + t;
                    if (p < P.N) {
                        const size_t rowi = ((size_t)bb * P.N + scan_to_token(p, P.H, P.W, P.dir)) * P.heads + hh;
                        prefetch_l2((i & 1) ? (const void *)(P.q + rowi * P.ldk) : (const void *)(P.g + rowi * P.ldk));
                    }
                }
            }
        }
        gc0 += (uint32_t)nch;
        __syncthreads();
        // the next sequence's first chunks land while this one's corrections run (the
        // staging slots are free: every chunk gated, the look-back slots read)
        if (warp == kWarpG && seq + ngrp < P.n_seq) load_head(A, sm, sbase, gc0, seq + ngrp, lane);

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
                        // all sixteen loads first (rows past the grid read the sequence's first
                        // token and are zeroed after), so that their latencies overlap
                        float2 gl[8];
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const int p = cabs * kChunk + t0 + u;
                            const int pc = p < P.N ? p : 0;
                            const size_t rowi = ((size_t)bb * P.N + scan_to_token(pc, P.H, P.W, P.dir)) * P.heads + hh;
                            gl[u] = ld_gate2<kZ>(reinterpret_cast<const uint8_t *>(P.g + rowi * P.ldk + 2 * lane), A.inv_tau);
                            qv[u] = *reinterpret_cast<const __half2 *>(P.q + rowi * P.ldk + 2 * lane);
                        }
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const bool ok = cabs * kChunk + t0 + u < P.N;
                            acc.x += ok ? gl[u].x : 0.f;
                            acc.y += ok ? gl[u].y : 0.f;
                            pg[u] = acc;
                            if (!ok) qv[u] = __float2half2_rn(0.f);
                        }
                        *reinterpret_cast<float2 *>(htot + gw * 64 + 2 * lane) = acc;
                        named_sync(kBarGAll, kGThreads);
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
                        named_sync(kBarGAll, kGThreads);   // htot reused by the next chunk
                    }
                    (void)tg;
                }
                fence_proxy_async_cta();
                __syncthreads();
                if (warp == kWarpRE) {
                    tc_fence_after();
                    if (elect_one_sync()) {
                        constexpr uint32_t id_o = idesc_f16_f32(64, kDV, false, true);
                        for (int li = 0; li < nl; ++li) {
                            const uint32_t ba = sbase + (batch == 0 ? held_tile(li) : L::vop + kTile);
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                umma_f16(tmem + 64 * li, desc_sw128(qaddr[li] + kk * 32, 16, 1024),
                                         desc_sw128(ba + kk * 2048, kTile, 1024), id_o, kk > 0 ? 1u : 0u);
                        }
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
                        // staging: the output tile for team 0, the first ring tile (free once the
                        // batch's products are complete) for team 1
                        add_out_tile(P, o, q4, lane, tb, sm + (team ? L::ring : L::ostg), rows,
                                     team ? kBarT1 : kBarT0);
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
    if (warp == kWarpU) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace pp
}  // namespace gtr
