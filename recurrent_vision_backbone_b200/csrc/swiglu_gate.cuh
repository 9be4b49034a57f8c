// swiglu_gate.cuh -- the gated value branch of GTR's Spatial SwiGLU for sm_100a
// (included by gtr_gla.cu, which holds the C ABI).
//
// GTR news article (tokendh.com), section "单向扫描的致命缺陷，以及GTR怎么补": Spatial
// SwiGLU puts a 3x3 depthwise convolution into the value branch of a SwiGLU, so that
// every patch sees its eight grid neighbours at once.  The fused step computed here,
// between the block's up/gate projections and its down projection (plain library
// GEMMs), is
//
//     h[b,y,x,c] = silu(G[b,y,x,c]) * (bias[c] + sum_{i,j<3} w[c][i][j] U[b,y+i-1,x+j-1,c])
//
// (cross-correlation, zero padding, silu(x) = x sigmoid(x)), G, U, h fp16 [B, H, W, C]
// with channels contiguous, w fp32 [C][3][3], bias fp32 [C] or absent.  One pass over
// the activations: read U and G once, write h once (6 bytes per element); HBM-bound.
//
// CTAs over 16x16-pixel, 64-channel tiles of the B x H x W x C grid (one tile per CTA,
// two CTAs per SM; a persistent two-stage variant, one CTA per SM, is kept as a
// tuning option — it measured slower):
//   * one thread issues, per tile, two TMA tensor copies into a stage: U with a
//     one-pixel halo (18x18 pixels; the copy's zero fill supplies the padding: loads
//     may start at coordinate -1) and G (16x16), completion on the stage's mbarrier
//     (bounded wait);
//   * 512 threads: thread = (channel pair, column); each slides a 3x3 window down its
//     column, three new U loads per row, packed fp32 FMAs (one partial sum per kernel
//     row), SiLU with __expf and a reciprocal, and writes h over the G it read (one
//     element, one thread);
//   * the same thread stores the tile with a TMA tensor copy (clipped at the grid's
//     edges) and, with more stages, refills the stage once the copy has read it.
// Shared memory rows are 128 bytes (64 channels): a warp (32 channel pairs of one
// pixel) reads 128 contiguous bytes, conflict-free.  73 KB per stage.
#pragma once

namespace gtr {
namespace sw {

constexpr int kTY = 16, kTX = 16, kTC = 64;   // tile rows, columns, channels
constexpr int kThreads = 512;
constexpr int kUBytes = (kTY + 2) * (kTX + 2) * kTC * 2;   // 41472
constexpr int kGBytes = kTY * kTX * kTC * 2;               // 32768
constexpr int kStageBytes = kUBytes + kGBytes;             // 74240 = 580 * 128
template <int NS>   // stages
struct L {
    static constexpr int stage = 0;                // [NS] U then G (h written over G)
    static constexpr int bar = NS * kStageBytes;   // [NS] stage landed
    static constexpr int bytes = bar + 8 * NS;
    static constexpr int alloc = bytes + 128;      // base alignment slack
};
static_assert(kUBytes % 128 == 0 && kStageBytes % 128 == 0, "TMA destination alignment");
static_assert(L<2>::alloc <= 227 * 1024, "two stages fit one CTA");

struct Args {
    CUtensorMap mu, mg, mh;   // U (box 64 x 18 x 18), G and h (box 64 x 16 x 16)
    const float *w, *bias;
    int B, H, W, C;
    int tiles_x, tiles_y, tiles_c, tiles;
};

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap *m, int c0, int c1, int c2, int c3,
                                            uint32_t mbar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, "
        "%4, %5}], [%6];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(mbar)
        : "memory");
}
__device__ __forceinline__ void tma_store_4d(const CUtensorMap *m, uint32_t src, int c0, int c1, int c2, int c3) {
    asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%1, %2, %3, %4}], [%5];" ::"l"(
                     reinterpret_cast<uint64_t>(m)),
                 "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(src)
                 : "memory");
}

__device__ __forceinline__ float silu_f(float x) { return x * __frcp_rn(1.f + __expf(-x)); }

struct Tile {
    int c0, x0, y0, b;
};
__device__ __forceinline__ Tile tile_of(const Args &A, int t) {
    Tile r;
    const int tc = t % A.tiles_c;
    t /= A.tiles_c;
    const int tx = t % A.tiles_x;
    t /= A.tiles_x;
    const int ty = t % A.tiles_y;
    r.b = t / A.tiles_y;
    r.c0 = tc * kTC;
    r.x0 = tx * kTX;
    r.y0 = ty * kTY;
    return r;
}

// The two copies of tile t into stage `st` (one thread).
__device__ __forceinline__ void load_tile(const Args &A, uint32_t sbase, uint64_t *bar, int st, int t) {
    const Tile T = tile_of(A, t);
    const uint32_t dst = sbase + st * kStageBytes;
    // the full boxes always arrive (out-of-grid parts as the copies' zero fill)
    mbar_arrive_expect_tx(bar + st, (uint32_t)kStageBytes);
    tma_load_4d(dst, &A.mu, T.c0, T.x0 - 1, T.y0 - 1, T.b, smem_u32(bar + st));
    tma_load_4d(dst + kUBytes, &A.mg, T.c0, T.x0, T.y0, T.b, smem_u32(bar + st));
}

// NS stages: 2 for persistent CTAs (one per SM, the next tile's copies in flight
// while a tile computes), 1 for one tile per CTA (two CTAs per SM).
template <int NS>
__global__ void __launch_bounds__(kThreads, 1) swiglu_gate_kernel(const __grid_constant__ Args A) {
    extern __shared__ uint8_t smem_raw[];
    // aligned by an offset from the shared array itself (not through an integer), so
    // that the compiler still sees every access as shared memory
    uint8_t *sm = smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u);
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + L<NS>::bar);
    const int tid = threadIdx.x;
    if (tid == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&A.mu)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&A.mg)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&A.mh)) : "memory");
        for (int s2 = 0; s2 < NS; ++s2) mbar_init(bar + s2, 1);
        fence_mbar_init();
    }
    __syncthreads();
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int t0 = blockIdx.x, dt = gridDim.x;
    int issued[NS];   // copies issued per stage (thread 0)
#pragma unroll
    for (int s2 = 0; s2 < NS; ++s2) {
        issued[s2] = 0;
        if (tid == 0 && t0 + s2 * dt < A.tiles) {
            load_tile(A, sbase, bar, s2, t0 + s2 * dt);
            ++issued[s2];
        }
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // this thread: channels cl, cl+1 of a tile, column x
    const int cp = tid & 31, x = tid >> 5;
    const int cl = 2 * cp;
    bool ok = true;
    float hmx = 0.f;
    int i = 0;
    for (int t = t0; t < A.tiles; t += dt, ++i) {
        const int st = i % NS;
        const Tile T = tile_of(A, t);
        const int c = T.c0 + cl;
        float2 wk[9];
#pragma unroll
        for (int k = 0; k < 9; ++k)
            wk[k] = make_float2(c < A.C ? A.w[(size_t)c * 9 + k] : 0.f, c + 1 < A.C ? A.w[(size_t)(c + 1) * 9 + k] : 0.f);
        float2 bs = make_float2(0.f, 0.f);
        if (A.bias != nullptr) bs = make_float2(c < A.C ? A.bias[c] : 0.f, c + 1 < A.C ? A.bias[c + 1] : 0.f);
        // one decision for the whole CTA (a thread whose wait ran out must not leave
        // the others at the barrier below)
        ok = __syncthreads_and(mbar_wait_bounded(bar + st, (uint32_t)(i / NS) & 1u, kWaitLimitNs)) != 0;
        if (!ok) {
            if (tid == 0) set_error(kErrTimeout);
            break;
        }
        const uint8_t *us = sm + st * kStageBytes;
        uint8_t *gs = sm + st * kStageBytes + kUBytes;
        // the window: U rows r, r+1, r+2 (halo coordinates) at columns x .. x+2
        float2 win[3][3];
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int j = 0; j < 3; ++j)
                win[r][j] = __half22float2(*reinterpret_cast<const __half2 *>(us + ((r * (kTX + 2) + x + j) * kTC + cl) * 2));
#pragma unroll 8
        for (int y = 0; y < kTY; ++y) {
#pragma unroll
            for (int j = 0; j < 3; ++j)
                win[2][j] = __half22float2(
                    *reinterpret_cast<const __half2 *>(us + (((y + 2) * (kTX + 2) + x + j) * kTC + cl) * 2));
            // both channels at once: packed fp32 FMAs (each lane still rounds in fp32),
            // one partial sum per kernel row so that the chains are three deep
            float2 pr[3];
#pragma unroll
            for (int r = 0; r < 3; ++r) {
                pr[r] = __fmul2_rn(wk[3 * r], win[r][0]);
#pragma unroll
                for (int j = 1; j < 3; ++j) pr[r] = __ffma2_rn(wk[3 * r + j], win[r][j], pr[r]);
            }
            const float2 acc = __fadd2_rn(__fadd2_rn(pr[0], pr[1]), __fadd2_rn(pr[2], bs));
            __half2 *gp = reinterpret_cast<__half2 *>(gs + ((y * kTX + x) * kTC + cl) * 2);
            const float2 gv = __half22float2(*gp);
            const float2 hv = __fmul2_rn(make_float2(silu_f(gv.x), silu_f(gv.y)), acc);
            const float h0 = hv.x, h1 = hv.y;
            hmx = fmaxf(hmx, fmaxf(fabsf(h0), fabsf(h1)));
            *gp = __floats2half2_rn(h0, h1);
#pragma unroll
            for (int j = 0; j < 3; ++j) {
                win[0][j] = win[1][j];
                win[1][j] = win[2][j];
            }
        }
        // the tile of h (written over G) to global memory: the async proxy reads it
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncthreads();
        if (tid == 0) {
            tma_store_4d(&A.mh, smem_u32(gs), T.c0, T.x0, T.y0, T.b);
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            // the stage is refilled only after the store has read it
            asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
            if (t + NS * dt < A.tiles) {
                load_tile(A, sbase, bar, st, t + NS * dt);
                ++issued[st];
            }
        }
    }
    range_check(hmx);
    if (tid == 0) {
        if (!ok) {
            // copies may still be in flight: the CTA's shared memory stays until this
            // thread exits, so it waits (bounded as well) for each stage's last phase
            for (int s2 = 0; s2 < NS; ++s2)
                if (issued[s2] > 0) mbar_wait_bounded(bar + s2, (uint32_t)(issued[s2] - 1) & 1u, kWaitLimitNs);
        }
        asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    }
}

}  // namespace sw
}  // namespace gtr
