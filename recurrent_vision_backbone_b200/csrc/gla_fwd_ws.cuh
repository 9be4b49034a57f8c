// gla_fwd_ws.cuh -- warp-specialised, round-pipelined variant of the GTR token-mixer
// forward kernel for dk = dv = 64 (included by gtr_gla.cu, which holds the shared
// helpers, the 128-key-channel kernel and the C ABI).
//
// Same mathematics and cluster decomposition as gla_fwd_kernel (one cluster of P CTAs
// per (batch, head) sequence, one 64-token chunk per CTA per round, element-sliced
// state pass over DSMEM), but each CTA runs two warp groups that work on different
// rounds at the same time:
//
//   group A (warps 0-7): waits for the bulk-copied raw rows of round R, builds the
//     gated operands, issues MMA 1 (state delta and scores), reads the scores and the
//     state delta out of TMEM, and announces round R's (d, dS) to every CTA of the
//     cluster;
//   group B (warps 8-11): runs the state pass of round R (reads every peer's (d, dS)
//     slice, writes S_prev into every peer's operand tile), issues MMA 2 (output) and
//     stores the outputs;
//   loader (warp 12): fetches the raw rows of upcoming rounds with 16-byte cp.async
//     into double-buffered staging and signals their arrival through an mbarrier
//     (cp.async.mbarrier.arrive); it never executes a fence, so loads in flight hold
//     up no other warp.
//
// Group A of round R only depends on group B of round R-2, so the gating, MMA 1 and
// readout of one round overlap the state pass, MMA 2 and output of the previous one.
// Round-to-round hand-offs are mbarrier pairs (full / empty) per double-buffered tile;
// cross-CTA ones are arrived remotely with release semantics at cluster scope and
// waited on with acquire semantics.
#pragma once

namespace gtr {
namespace ws {

constexpr int kThreadsA = 256;          // warps 0-7
constexpr int kThreadsB = 128;          // warps 8-11
constexpr int kThreads = kThreadsA + kThreadsB + 32;   // + loader warp 12
constexpr int kDK = 64;
constexpr uint32_t kBarA = 1, kBarB = 2;   // named barrier ids
constexpr int kMaxM = 4;                   // state float4 per group-B thread (cluster size >= 2)
constexpr int kMinCluster = 2;

// ------------------------------------------------------------------ smem map
struct L {
    static constexpr int stg = 0;                  // raw rows q,k,g,v, unswizzled [64][128 B] x 4, x2
    static constexpr int stg_bytes = 4 * kTile;
    static constexpr int qint = stg + 2 * stg_bytes;   // Q * P (or Q * pi * before), x2
    static constexpr int kt = qint + 2 * kTile;       // K / P (or K * sigma * after)
    static constexpr int vop = kt + kTile;            // V, swizzled, x2
    static constexpr int p = vop + 2 * kTile;         // masked scores, x2
    static constexpr int qj = p + 2 * kTile;          // packed Q^(J) (sub-block path)
    static constexpr int qj_bytes = (64 + 48 + 32 + 16) * 128;
    static constexpr int kbar = qj + qj_bytes;        // K * sigma (sub-block path)
    static constexpr int sop = kbar + kTile;          // S_prev fp16, x2
    static constexpr int agg = sop + 2 * kTile;       // dS fp32 [64][64] swizzled, x2
    static constexpr int ost = agg + 2 * 64 * 256;    // output staging (group B)
    static constexpr int dvec = ost + kTile;          // d of the chunk [64] fp32, x2
    static constexpr int dloc = dvec + 2 * 256;       // d, local copy for the readout
    static constexpr int htot = dloc + 256;           // half-block totals [8][64]
    static constexpr int diag = htot + 8 * 64 * 4;    // exact diagonal blocks [4][16][16]
    static constexpr int rowb = diag + 4 * 16 * 16 * 4;   // group-B token rows [64]
    static constexpr int misc = rowb + 64 * 4;
    // misc, per round parity: flags[4], max |q| per sub-block [4], max |k|  (48 bytes each)
    static constexpr int bars = misc + 128;
    static constexpr int bytes = bars + 24 * 8 + 16;
    static constexpr int alloc = bytes + 1024;

    static __host__ __device__ constexpr int qj_region(int J) {
        return 128 * (J == 0 ? 0 : J == 1 ? 64 : J == 2 ? 112 : 144);
    }
};
static_assert(L::alloc <= 227 * 1024, "shared memory budget");

// barrier slots (uint64_t index inside L::bars)
enum {
    B_STG = 0,        // [2]  raw rows landed (tx bytes)
    B_MMA1 = 2,       //      MMA 1 complete
    B_MMA2 = 3,       //      MMA 2 complete
    B_OPSF = 4,       // [2]  Qint / P / V of round R ready for MMA 2 (group A -> B)
    B_OPSE = 6,       // [2]  MMA 2 of round R done with them (group B -> A)
    B_AGGF = 8,       // [2]  every CTA's (d, dS) of round R written (P remote arrivals)
    B_AGGE = 10,      // [2]  every scan owner done reading this CTA's (d, dS)
    B_SOPF = 12,      // [2]  every scan owner wrote its slice of this CTA's S_prev
    B_SOPE = 14,      // [2]  every CTA's MMA 2 done with its S_prev tile
    B_STGE = 16,      // [2]  group A done with the raw rows of a staging buffer
    B_TMEM = 18       //      (uint32_t) TMEM base address
};

struct Sched {
    int n_rounds_seq;   // rounds per sequence
    int cl, ncl, rank, CP;
    int n_seq, n_chunks;
    __device__ int total() const {
        const int nseq_local = cl < n_seq ? (n_seq - cl + ncl - 1) / ncl : 0;
        return nseq_local * n_rounds_seq;
    }
    // round R -> sequence, round inside the sequence, chunk
    __device__ void at(int R, int &seq, int &rr, int &c) const {
        const int s = R / n_rounds_seq;
        rr = R - s * n_rounds_seq;
        seq = cl + s * ncl;
        c = rr * CP + rank;
    }
};

__device__ __forceinline__ uint64_t *bar(uint8_t *sm, int i) {
    return reinterpret_cast<uint64_t *>(sm + L::bars) + i;
}

__device__ __forceinline__ bool wait_local(uint64_t *b, uint32_t parity, bool &to) {
    if (!mbar_wait_bounded(b, parity, kWaitLimitNs)) {
        to = true;
        set_error(kErrTimeout);
        return false;
    }
    return true;
}
__device__ __forceinline__ bool wait_cluster(uint64_t *b, uint32_t parity, bool &to) {
    if (!mbar_wait_cluster_bounded(b, parity, kWaitLimitNs)) {
        to = true;
        set_error(kErrTimeout);
        return false;
    }
    return true;
}

// Loader warp: 16-byte cp.async of the 64 rows of chunk c of sequence seq (q, k, g, v)
// into staging s; rows past the end of the grid are zero-filled.  Completion is
// signalled on the staging barrier by every lane (32 arrivals).
__device__ __forceinline__ void load_rows(const Params &P, uint8_t *sm, int seq, int c, int s,
                                          int lane) {
    const uint32_t st = smem_u32(sm + L::stg + s * L::stg_bytes);
    const int b = seq / P.heads, h = seq - b * P.heads;
    const int p0 = c * kChunk;
    // lane covers rows lane and lane + 32; 8 pieces of 16 B per row per tensor
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int t = lane + 32 * half;
        const bool ok = p0 + t < P.N;
        size_t ro = 0;
        if (ok) ro = (size_t)((b * P.N + scan_to_token(p0 + t, P.H, P.W, P.dir)) * P.heads + h);
        const uint32_t nb = ok ? 16u : 0u;
        const __half *src[4] = {P.q + ro * kDK, P.k + ro * kDK, P.g + ro * kDK, P.v + ro * kDV};
#pragma unroll
        for (int ten = 0; ten < 4; ++ten)
#pragma unroll
            for (int pc = 0; pc < 8; ++pc)
                cp_async16(st + ten * kTile + t * 128 + 16 * pc, src[ten] + 8 * pc, nb);
    }
    cp_async_mbar_arrive_noinc(bar(sm, B_STG + s));
}

__global__ void __launch_bounds__(kThreads, 1) gla_fwd_ws_kernel(const Params P) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    Sched sc;
    sc.rank = (int)cluster_ctarank();
    sc.ncl = (int)nclusters_x();
    sc.CP = (int)(gridDim.x / (unsigned)sc.ncl);
    sc.cl = (int)cluster_id_x();
    sc.n_seq = P.n_seq;
    sc.n_chunks = P.n_chunks;
    sc.n_rounds_seq = (P.n_chunks + sc.CP - 1) / sc.CP;
    const int CP = sc.CP, rank = sc.rank;
    const int total = sc.total();

    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar(sm, B_TMEM));

    if (warp == 0) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar(sm, B_STG), 32);
        mbar_init(bar(sm, B_STG + 1), 32);
        mbar_init(bar(sm, B_STGE), 1);
        mbar_init(bar(sm, B_STGE + 1), 1);
        mbar_init(bar(sm, B_MMA1), 1);
        mbar_init(bar(sm, B_MMA2), 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(sm, B_OPSF + i), 1);
            mbar_init(bar(sm, B_OPSE + i), 1);
            mbar_init(bar(sm, B_AGGF + i), (uint32_t)CP);
            mbar_init(bar(sm, B_AGGE + i), (uint32_t)CP);
            mbar_init(bar(sm, B_SOPF + i), (uint32_t)CP);
            mbar_init(bar(sm, B_SOPE + i), (uint32_t)CP);
        }
        fence_mbar_init();
    }
    if (tid < 24) reinterpret_cast<unsigned *>(sm + L::misc)[(tid / 12) * 12 + tid % 12] = 0u;
    tc_fence_before();
    __syncthreads();
    cluster_sync();   // every CTA's barriers are initialised before any remote arrive
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool to = false;

    if (warp < 8) {
        // ======================================================= group A
        const int gI = warp >> 1, ghf = warp & 1, gt0 = 16 * gI + 8 * ghf, gh = 2 * gI + ghf;
        const int sp = warp & 3, chalf = warp >> 2;
        const int rrow0 = 16 * sp + (lane >> 2);
        const int rcol0 = 32 * chalf + 2 * (lane & 3);
        float *htot = reinterpret_cast<float *>(sm + L::htot);
        float *dloc = reinterpret_cast<float *>(sm + L::dloc);
        float *diagx = reinterpret_cast<float *>(sm + L::diag);
        uint32_t n_mma1 = 0;
        uint32_t vuse[2] = {0u, 0u};   // valid rounds seen per buffer (ops barriers)
        for (int R = 0; R < total; ++R) {
            int seq, rr, c;
            sc.at(R, seq, rr, c);
            const bool valid = c < P.n_chunks;
            const int b = R & 1;
            const uint32_t k = (uint32_t)(R >> 1);
            const int nrows = valid ? min(kChunk, P.N - c * kChunk) : 0;
            const uint8_t *st = sm + L::stg + b * L::stg_bytes;
            int *flags = reinterpret_cast<int *>(sm + L::misc + 48 * b);
            unsigned *qmax = reinterpret_cast<unsigned *>(sm + L::misc + 48 * b + 16);
            unsigned *kmax = reinterpret_cast<unsigned *>(sm + L::misc + 48 * b + 32);
            bool slow = false;
            if (valid) {
                wait_local(bar(sm, B_STG + b), vuse[b] & 1u, to);
                wait_local(bar(sm, B_OPSE + b), (vuse[b] & 1u) ^ 1u, to);
                // ---------- pass 1: a = exp(g), half-block products; q, k to registers
                float pl[8][2], sl[8][2];
                __half2 qh[8], kh[8];
                float qm = 0.f, km = 0.f;
                {
                    float a0[8], a1[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int t = gt0 + u;
                        const uint32_t o = t * 128 + 4 * lane;
                        float2 gv = make_float2(0.f, 0.f);
                        qh[u] = __float2half2_rn(0.f);
                        kh[u] = __float2half2_rn(0.f);
                        if (t < nrows) {
                            gv = ld_h2(st + 2 * kTile + o);
                            qh[u] = *reinterpret_cast<const __half2 *>(st + o);
                            kh[u] = *reinterpret_cast<const __half2 *>(st + kTile + o);
                        }
                        a0[u] = exp_f(gv.x);
                        a1[u] = exp_f(gv.y);
                        const __half2 qa = __habs2(qh[u]), ka = __habs2(kh[u]);
                        qm = fmaxf(qm, fmaxf(__low2float(qa), __high2float(qa)));
                        km = fmaxf(km, fmaxf(__low2float(ka), __high2float(ka)));
                    }
                    float r0 = 1.f, r1 = 1.f;
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        r0 *= a0[u]; r1 *= a1[u];
                        pl[u][0] = r0; pl[u][1] = r1;
                    }
                    r0 = 1.f; r1 = 1.f;
#pragma unroll
                    for (int u = 7; u >= 0; --u) {
                        sl[u][0] = r0; sl[u][1] = r1;
                        r0 *= a0[u]; r1 *= a1[u];
                    }
                    *reinterpret_cast<float2 *>(htot + gh * 64 + 2 * lane) = make_float2(pl[7][0], pl[7][1]);
                }
                {
                    const unsigned wq = __reduce_max_sync(0xffffffffu, __float_as_uint(qm));
                    const unsigned wk = __reduce_max_sync(0xffffffffu, __float_as_uint(km));
                    if (lane == 0) {
                        atomicMax(&qmax[gI], wq);
                        atomicMax(kmax, wk);
                    }
                }
                // V rows -> swizzled operand tile (zeros past the grid)
                {
                    uint8_t *vo = sm + L::vop + b * kTile;
#pragma unroll
                    for (int x = tid; x < 64 * 8; x += kThreadsA) {
                        const int t = x >> 3, c8 = x & 7;
                        uint4 val = make_uint4(0u, 0u, 0u, 0u);
                        if (t < nrows) val = *reinterpret_cast<const uint4 *>(st + 3 * kTile + t * 128 + 16 * c8);
                        *reinterpret_cast<uint4 *>(vo + sw_off(t, 8 * c8)) = val;
                    }
                }
                named_sync(kBarA, kThreadsA);
                // ---------- chunk factors for my two channels
                float dch[2], bef[2], aft[2];
                bool bad = __uint_as_float(*kmax) > kFastMaxK;
                {
                    float2 ht[8];
#pragma unroll
                    for (int h8 = 0; h8 < 8; ++h8)
                        ht[h8] = *reinterpret_cast<const float2 *>(htot + h8 * 64 + 2 * lane);
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
                        dch[e] = d; bef[e] = bf; aft[e] = af;
                        bad |= !(d >= kFastMinDecay);
                    }
                }
                slow = named_sync_or(kBarA, kThreadsA, bad);
                if (gh == 0) *reinterpret_cast<float2 *>(dloc + 2 * lane) = make_float2(dch[0], dch[1]);
                uint8_t *qo = sm + L::qint + b * kTile;
                if (!slow) {
                    const float i0 = aft[0] / dch[0], i1 = aft[1] / dch[1];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const uint32_t o = sw_off(gt0 + u, 2 * lane);
                        const float2 qv = __half22float2(qh[u]);
                        const float2 kv = __half22float2(kh[u]);
                        st_h2(qo + o, qv.x * (pl[u][0] * bef[0]), qv.y * (pl[u][1] * bef[1]));
                        st_h2(sm + L::kt + o, kv.x * (sl[u][0] * i0), kv.y * (sl[u][1] * i1));
                    }
                } else {
                    // sub-block path: off-diagonal factors are products of a's <= 1
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
                                        lg += __half2float(*reinterpret_cast<const __half *>(st + 2 * kTile + r2 * 128 + 2 * i));
                                    const float qv = __half2float(*reinterpret_cast<const __half *>(st + tu * 128 + 2 * i));
                                    const float kv = __half2float(*reinterpret_cast<const __half *>(st + kTile + tw * 128 + 2 * i));
                                    acc += qv * kv * exp_f(lg);
                                }
                            }
                            diagx[(I * 16 + u) * 16 + w] = acc;
                        }
                        named_sync(kBarA, kThreadsA);
                    }
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
                        bI[e] = b0; aI[e] = a0;
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
                        st_h2(sm + L::kbar + o, ks0, ks1);
                        st_h2(sm + L::kt + o, ks0 * aI[0], ks1 * aI[1]);
#pragma unroll
                        for (int J = 0; J < 4; ++J) {
                            if (J <= gI) {
                                const int rows_j = 64 - 16 * J;
                                (void)rows_j;
                                st_h2(sm + L::qj + L::qj_region(J) + sw_off(t - 16 * J, 2 * lane),
                                      qp0 * cf[0][J], qp1 * cf[1][J]);
                            }
                        }
                    }
                }
                fence_proxy_async_cta();
                named_sync(kBarA, kThreadsA);
                // raw rows of this staging buffer are consumed: the loader may refill it
                if (tid == 0) mbar_arrive(bar(sm, B_STGE + b));
                // ---------- MMA 1
                if (tid == 0) {
                    tc_fence_after();
                    const uint32_t kta = sbase + L::kt;
                    const uint32_t va = sbase + L::vop + b * kTile;
                    constexpr uint32_t id_ds = idesc_f16_f32(64, kDV, true, true);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16(tmem + 0, desc_sw128(kta + kk * 2048, kTile, 1024),
                                 desc_sw128(va + kk * 2048, kTile, 1024), id_ds, kk > 0 ? 1u : 0u);
                    if (!slow) {
                        constexpr uint32_t id = idesc_f16_f32(64, 64, false, false);
                        const uint32_t qa = sbase + L::qint + b * kTile;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_f16(tmem + 64, desc_sw128(qa + kk * 32, 16, 1024),
                                     desc_sw128(kta + kk * 32, 16, 1024), id, kk > 0 ? 1u : 0u);
                    } else {
                        constexpr uint32_t id = idesc_f16_f32(64, 16, false, false);
                        for (int J = 0; J < 4; ++J) {
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                const uint32_t aa = sbase + L::qj + L::qj_region(J) - 16 * J * 128 + kk * 32;
                                const uint32_t bb = sbase + L::kbar + 16 * J * 128 + kk * 32;
                                umma_f16(tmem + 64 + 16 * J, desc_sw128(aa, 16, 1024),
                                         desc_sw128(bb, 16, 1024), id, kk > 0 ? 1u : 0u);
                            }
                        }
                    }
                    umma_commit(bar(sm, B_MMA1));
                }
                wait_local(bar(sm, B_MMA1), n_mma1 & 1u, to);
                ++n_mma1;
                tc_fence_after();
                uint32_t rs[16], rd[16];
                tmem_ld_16x256b_x4(tmem + ((uint32_t)(32 * sp) << 16) + 64 + 32 * chalf, rs);
                tmem_ld_16x256b_x4(tmem + ((uint32_t)(32 * sp) << 16) + 32 * chalf, rd);
                tmem_ld_wait();
                // scores -> masked fp16 P
                {
                    uint8_t *pt = sm + L::p + b * kTile;
                    const bool fb = slow && (flags[sp] != 0);
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const int row = rrow0 + 8 * hh;
                            const int col = rcol0 + 8 * cc;
                            float x0 = __uint_as_float(rs[4 * cc + 2 * hh]);
                            float x1 = __uint_as_float(rs[4 * cc + 2 * hh + 1]);
                            if (fb && (col >> 4) == sp) {
                                x0 = diagx[(sp * 16 + (row & 15)) * 16 + (col & 15)];
                                x1 = diagx[(sp * 16 + (row & 15)) * 16 + ((col + 1) & 15)];
                            }
                            x0 = col <= row ? x0 : 0.f;
                            x1 = col + 1 <= row ? x1 : 0.f;
                            st_h2(pt + sw_off(row, col), x0, x1);
                        }
                    }
                }
                tc_fence_before();
                // every scan owner must be done with this CTA's (d, dS) of round R-2
                wait_cluster(bar(sm, B_AGGE + b), (k & 1u) ^ 1u, to);
                {
                    uint8_t *ag = sm + L::agg + b * (64 * 256);
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int i = rrow0 + 8 * hh;
                        const float scl = slow ? 1.f : dloc[i];
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc) {
                            const int col = rcol0 + 8 * cc;
                            *reinterpret_cast<float2 *>(ag + agg_off(i, col >> 2) + (col & 3) * 4) =
                                make_float2(scl * __uint_as_float(rd[4 * cc + 2 * hh]),
                                            scl * __uint_as_float(rd[4 * cc + 2 * hh + 1]));
                        }
                    }
                    if (tid < 64) reinterpret_cast<float *>(sm + L::dvec + b * 256)[tid] = dloc[tid];
                }
                fence_proxy_async_cta();
                named_sync(kBarA, kThreadsA);
                // flags / maxima of this parity are next used two rounds later, after
                // every group-A thread has passed the next round's barriers
                if (tid < 4) { flags[tid] = 0; qmax[tid] = 0u; }
                if (tid == 0) {
                    *kmax = 0u;
                    mbar_arrive(bar(sm, B_OPSF + b));
                }
                // one remote arrive per thread: the release fences run in parallel
                if (tid >= 32 && tid < 32 + CP)
                    mbar_arrive_remote(smem_u32(bar(sm, B_AGGF + b)), (uint32_t)(tid - 32));
                ++vuse[b];
            } else {
                // no chunk for this CTA this round: keep the cluster protocol in step
                wait_cluster(bar(sm, B_AGGE + b), (k & 1u) ^ 1u, to);
                named_sync(kBarA, kThreadsA);
                if (tid < CP) mbar_arrive_remote(smem_u32(bar(sm, B_AGGF + b)), (uint32_t)tid);
            }
        }
    } else if (warp < 12) {
        // ======================================================= group B
        const int tb = tid - kThreadsA;         // 0..127
        const int bw = warp - 8;                 // 0..3 (TMEM subpartition)
        int *rowb = reinterpret_cast<int *>(sm + L::rowb);
        const int NF4 = kDK * kDV / 4;
        const int slo = (int)((long)rank * NF4 / CP);
        const int shi = (int)((long)(rank + 1) * NF4 / CP);
        const int nloc = shi - slo;
        uint32_t n_mma2 = 0;
        uint32_t vuse[2] = {0u, 0u};
        float4 S[kMaxM];
        for (int R = 0; R < total; ++R) {
            int seq, rr, c;
            sc.at(R, seq, rr, c);
            const bool valid = c < P.n_chunks;
            const int b = R & 1;
            const uint32_t k = (uint32_t)(R >> 1);
            const int nvalid = min(CP, P.n_chunks - rr * CP);
            if (rr == 0) {
#pragma unroll
                for (int m = 0; m < kMaxM; ++m) {
                    const int el = tb + m * kThreadsB;
                    S[m] = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (P.s0 != nullptr && el < nloc)
                        S[m] = reinterpret_cast<const float4 *>(P.s0 + (size_t)seq * kDK * kDV)[slo + el];
                }
            }
            // ---------- state pass over the round's chunks
            wait_cluster(bar(sm, B_AGGF + b), k & 1u, to);
            wait_cluster(bar(sm, B_SOPE + b), (k & 1u) ^ 1u, to);
            {
                const uint32_t agg_b = sbase + L::agg + b * (64 * 256);
                const uint32_t dv_b = sbase + L::dvec + b * 256;
                const uint32_t sop_b = sbase + L::sop + b * kTile;
                if (nvalid == 1) {
                    // one chunk in the round (cluster size 1 or a short last round):
                    // fetch four elements' (d, dS) at a time, then chain
#pragma unroll
                    for (int m0 = 0; m0 < kMaxM; m0 += 4) {
                        float4 a4[4];
                        float dd[4];
#pragma unroll
                        for (int mm = 0; mm < 4; ++mm) {
                            const int el = tb + (m0 + mm) * kThreadsB;
                            if (el < nloc) {
                                const int e = slo + el, i = e >> 4, c4 = e & 15;
                                a4[mm] = ld_dsmem_f4(mapa(agg_b + agg_off(i, c4), 0u));
                                dd[mm] = ld_dsmem_f32(mapa(dv_b + i * 4, 0u));
                            }
                        }
#pragma unroll
                        for (int mm = 0; mm < 4; ++mm) {
                            const int m = m0 + mm;
                            const int el = tb + m * kThreadsB;
                            if (el < nloc) {
                                const int e = slo + el, i = e >> 4, c4 = e & 15;
                                st_dsmem_v2(mapa(sop_b + sw_off(i, 4 * c4), 0u), pack_half2(S[m].x, S[m].y),
                                            pack_half2(S[m].z, S[m].w));
                                S[m].x = fmaf(dd[mm], S[m].x, a4[mm].x);
                                S[m].y = fmaf(dd[mm], S[m].y, a4[mm].y);
                                S[m].z = fmaf(dd[mm], S[m].z, a4[mm].z);
                                S[m].w = fmaf(dd[mm], S[m].w, a4[mm].w);
                            }
                        }
                    }
                } else {
#pragma unroll
                    for (int m = 0; m < kMaxM; ++m) {
                        const int el = tb + m * kThreadsB;
                        if (el < nloc) {
                            const int e = slo + el, i = e >> 4, c4 = e & 15;
                            const uint32_t aoff = agg_b + agg_off(i, c4);
                            const uint32_t doff = dv_b + i * 4;
                            const uint32_t soff = sop_b + sw_off(i, 4 * c4);
                            for (int j0 = 0; j0 < nvalid; j0 += 8) {
                                float4 a4[8];
                                float dd[8];
#pragma unroll
                                for (int q8 = 0; q8 < 8; ++q8) {
                                    if (j0 + q8 < nvalid) {
                                        a4[q8] = ld_dsmem_f4(mapa(aoff, (uint32_t)(j0 + q8)));
                                        dd[q8] = ld_dsmem_f32(mapa(doff, (uint32_t)(j0 + q8)));
                                    }
                                }
#pragma unroll
                                for (int q8 = 0; q8 < 8; ++q8) {
                                    if (j0 + q8 < nvalid) {
                                        st_dsmem_v2(mapa(soff, (uint32_t)(j0 + q8)),
                                                    pack_half2(S[m].x, S[m].y), pack_half2(S[m].z, S[m].w));
                                        S[m].x = fmaf(dd[q8], S[m].x, a4[q8].x);
                                        S[m].y = fmaf(dd[q8], S[m].y, a4[q8].y);
                                        S[m].z = fmaf(dd[q8], S[m].z, a4[q8].z);
                                        S[m].w = fmaf(dd[q8], S[m].w, a4[q8].w);
                                    }
                                }
                            }
                        }
                    }
                }
            }
            fence_proxy_async_cluster();
            named_sync(kBarB, kThreadsB);
            // peers may overwrite their (d, dS) of this buffer; my slice of every S_prev
            // tile is written (one remote arrive per thread)
            if (tb < CP) mbar_arrive_remote(smem_u32(bar(sm, B_AGGE + b)), (uint32_t)tb);
            if (tb >= 32 && tb < 32 + CP) mbar_arrive_remote(smem_u32(bar(sm, B_SOPF + b)), (uint32_t)(tb - 32));
            if (rr == sc.n_rounds_seq - 1 && P.sf != nullptr) {
#pragma unroll
                for (int m = 0; m < kMaxM; ++m) {
                    const int el = tb + m * kThreadsB;
                    if (el < nloc)
                        reinterpret_cast<float4 *>(P.sf + (size_t)seq * kDK * kDV)[slo + el] = S[m];
                }
            }
            // ---------- MMA 2 and the output rows
            wait_cluster(bar(sm, B_SOPF + b), k & 1u, to);
            if (valid) {
                // token rows of this chunk for the output store
                if (tb < 64) {
                    const int p = c * kChunk + tb;
                    int ro = -1;
                    if (p < P.N) {
                        const int bb = seq / P.heads, hh = seq - bb * P.heads;
                        ro = (bb * P.N + scan_to_token(p, P.H, P.W, P.dir)) * P.heads + hh;
                    }
                    rowb[tb] = ro;
                }
                wait_local(bar(sm, B_OPSF + b), vuse[b] & 1u, to);
                if (tb == 0) {
                    tc_fence_after();
                    constexpr uint32_t id = idesc_f16_f32(64, kDV, false, true);
                    const uint32_t qa = sbase + L::qint + b * kTile;
                    const uint32_t sa = sbase + L::sop + b * kTile;
                    const uint32_t pa = sbase + L::p + b * kTile;
                    const uint32_t va = sbase + L::vop + b * kTile;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16(tmem + 128, desc_sw128(qa + kk * 32, 16, 1024),
                                 desc_sw128(sa + kk * 2048, kTile, 1024), id, kk > 0 ? 1u : 0u);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16(tmem + 128, desc_sw128(pa + kk * 32, 16, 1024),
                                 desc_sw128(va + kk * 2048, kTile, 1024), id, 1u);
                    umma_commit(bar(sm, B_MMA2));
                }
                wait_local(bar(sm, B_MMA2), n_mma2 & 1u, to);
                ++n_mma2;
                ++vuse[b];
                tc_fence_after();
                if (tb == 0) mbar_arrive(bar(sm, B_OPSE + b));   // Qint / P / V of this buffer free
                {
                    uint32_t r0[16], r1[16];
                    const uint32_t ta = tmem + ((uint32_t)(32 * bw) << 16) + 128;
                    tmem_ld_16x256b_x4(ta, r0);
                    tmem_ld_16x256b_x4(ta + 32, r1);
                    tmem_ld_wait();
                    const int row0 = 16 * bw + (lane >> 2);
                    const int col0 = 2 * (lane & 3);
                    uint8_t *os = sm + L::ost;
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc)
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            st_h2(os + sw_off(row0 + 8 * hh, col0 + 8 * cc),
                                  __uint_as_float(r0[4 * cc + 2 * hh]), __uint_as_float(r0[4 * cc + 2 * hh + 1]));
                            st_h2(os + sw_off(row0 + 8 * hh, 32 + col0 + 8 * cc),
                                  __uint_as_float(r1[4 * cc + 2 * hh]), __uint_as_float(r1[4 * cc + 2 * hh + 1]));
                        }
                }
                tc_fence_before();
                named_sync(kBarB, kThreadsB);
#pragma unroll
                for (int x = tb; x < 64 * 8; x += kThreadsB) {
                    const int row = x >> 3, c8 = x & 7;
                    const int ro = rowb[row];
                    if (ro >= 0)
                        *reinterpret_cast<uint4 *>(P.out + (size_t)ro * kDV + 8 * c8) =
                            *reinterpret_cast<const uint4 *>(sm + L::ost + sw_off(row, 8 * c8));
                }
                named_sync(kBarB, kThreadsB);   // staging and row table reusable
            }
            if (tb >= 64 && tb < 64 + CP)   // this CTA is done with S_prev tile b
                mbar_arrive_remote(smem_u32(bar(sm, B_SOPE + b)), (uint32_t)(tb - 64));
        }
        // final states of sequences with no rounds (empty grid)
        if (total == 0 || sc.n_rounds_seq == 0) {
            for (int seq = sc.cl; seq < P.n_seq; seq += sc.ncl) {
                for (int el = tb; el < nloc; el += kThreadsB) {
                    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (P.s0 != nullptr) v = reinterpret_cast<const float4 *>(P.s0 + (size_t)seq * kDK * kDV)[slo + el];
                    if (P.sf != nullptr) reinterpret_cast<float4 *>(P.sf + (size_t)seq * kDK * kDV)[slo + el] = v;
                }
            }
        }
    } else {
        // ======================================================= loader (warp 12)
        uint32_t vuse[2] = {0u, 0u};
        for (int R = 0; R < total; ++R) {
            int seq, rr, c;
            sc.at(R, seq, rr, c);
            if (c >= P.n_chunks) continue;
            const int b = R & 1;
            // group A must be done with this staging buffer's previous rows
            wait_local(bar(sm, B_STGE + b), (vuse[b] & 1u) ^ 1u, to);
            load_rows(P, sm, seq, c, b, lane);
            ++vuse[b];
        }
        cp_async_wait_all();
    }

    __syncthreads();
    if (to) {
        // let any MMA still in flight finish before the shared memory and TMEM go away
        mbar_wait_bounded(bar(sm, B_MMA1), 0, kWaitLimitNs);
    }
    cluster_sync();   // no CTA leaves while a peer may still touch its shared memory
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace ws
}  // namespace gtr
