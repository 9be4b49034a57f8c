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
// One CTA per 16x16-pixel, 64-channel tile (a grid of them over B x H x W x C):
//   * one thread issues two TMA tensor copies: U with a one-pixel halo (18x18 pixels,
//     the copy's zero fill supplies the padding: loads may start at coordinate -1) and
//     G (16x16), completion on one mbarrier (bounded wait);
//   * 256 threads: thread = (channel pair, column pair); each slides a 3x3 window down
//     its two columns, three new U loads per row, fp32 math, SiLU with __expf and a
//     reciprocal, and writes h over the G it read (one element, one thread);
//   * one thread stores the tile with a TMA tensor copy (clipped at the grid's edges).
// Shared memory rows are 128 bytes (64 channels): a warp (32 channel pairs of one
// pixel) reads 128 contiguous bytes, conflict-free.  ~74 KB per CTA: three CTAs per SM.
#pragma once

namespace gtr {
namespace sw {

constexpr int kTY = 16, kTX = 16, kTC = 64;   // tile rows, columns, channels
constexpr int kThreads = 256;
constexpr int kUBytes = (kTY + 2) * (kTX + 2) * kTC * 2;   // 41472
constexpr int kGBytes = kTY * kTX * kTC * 2;               // 32768
struct L {
    static constexpr int u = 0;
    static constexpr int g = kUBytes;             // 128-byte aligned (41472 = 324 * 128)
    static constexpr int bar = g + kGBytes;
    static constexpr int bytes = bar + 16;
    static constexpr int alloc = bytes + 128;     // base alignment slack
};
static_assert(L::g % 128 == 0, "TMA destination alignment");

struct Args {
    CUtensorMap mu, mg, mh;   // U (box 64 x 18 x 18), G and h (box 64 x 16 x 16)
    const float *w, *bias;
    int B, H, W, C;
    int tiles_x, tiles_y, tiles_c;
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

__global__ void __launch_bounds__(kThreads) swiglu_gate_kernel(const __grid_constant__ Args A) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + L::bar);
    const int tid = threadIdx.x;
    int t = blockIdx.x;
    const int tc = t % A.tiles_c;
    t /= A.tiles_c;
    const int tx = t % A.tiles_x;
    t /= A.tiles_x;
    const int ty = t % A.tiles_y;
    const int b = t / A.tiles_y;
    const int c0 = tc * kTC, x0 = tx * kTX, y0 = ty * kTY;
    if (tid == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&A.mu)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&A.mg)) : "memory");
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (tid == 0) {
        // the full boxes always arrive (out-of-grid parts as the copies' zero fill)
        mbar_arrive_expect_tx(bar, (uint32_t)(kUBytes + kGBytes));
        tma_load_4d(sbase + L::u, &A.mu, c0, x0 - 1, y0 - 1, b, smem_u32(bar));
        tma_load_4d(sbase + L::g, &A.mg, c0, x0, y0, b, smem_u32(bar));
    }
    // this thread: channels cl, cl+1 of the tile, columns xa and xa + 8
    const int cp = tid & 31, xa = tid >> 5;
    const int cl = 2 * cp, c = c0 + cl;
    float2 wk[9];
    float2 bs = make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < 9; ++k) {
        const float w0 = c < A.C ? A.w[(size_t)c * 9 + k] : 0.f;
        const float w1 = c + 1 < A.C ? A.w[(size_t)(c + 1) * 9 + k] : 0.f;
        wk[k] = make_float2(w0, w1);
    }
    if (A.bias != nullptr) bs = make_float2(c < A.C ? A.bias[c] : 0.f, c + 1 < A.C ? A.bias[c + 1] : 0.f);
    const bool ok = mbar_wait_bounded(bar, 0, kWaitLimitNs);
    if (!ok) {
        set_error(kErrTimeout);
        // the copies may still be in flight: give them time before the CTA's shared
        // memory goes away (bounded as well)
        mbar_wait_bounded(bar, 0, kWaitLimitNs);
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (ok) {
        const uint8_t *us = sm + L::u;
        uint8_t *gs = sm + L::g;
        float hmx = 0.f;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int x = xa + 8 * half;   // output column in the tile; U columns x .. x+2
            // the window: U rows r, r+1, r+2 (halo coordinates) at columns x .. x+2
            float2 win[3][3];
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
                for (int j = 0; j < 3; ++j)
                    win[r][j] = __half22float2(*reinterpret_cast<const __half2 *>(
                        us + ((r * (kTX + 2) + x + j) * kTC + cl) * 2));
#pragma unroll 4
            for (int y = 0; y < kTY; ++y) {
#pragma unroll
                for (int j = 0; j < 3; ++j)
                    win[2][j] = __half22float2(*reinterpret_cast<const __half2 *>(
                        us + (((y + 2) * (kTX + 2) + x + j) * kTC + cl) * 2));
                float2 acc = bs;
#pragma unroll
                for (int i = 0; i < 3; ++i)
#pragma unroll
                    for (int j = 0; j < 3; ++j) {
                        acc.x = fmaf(wk[3 * i + j].x, win[i][j].x, acc.x);
                        acc.y = fmaf(wk[3 * i + j].y, win[i][j].y, acc.y);
                    }
                __half2 *gp = reinterpret_cast<__half2 *>(gs + ((y * kTX + x) * kTC + cl) * 2);
                const float2 gv = __half22float2(*gp);
                const float h0 = silu_f(gv.x) * acc.x, h1 = silu_f(gv.y) * acc.y;
                hmx = fmaxf(hmx, fmaxf(fabsf(h0), fabsf(h1)));
                *gp = __floats2half2_rn(h0, h1);
#pragma unroll
                for (int j = 0; j < 3; ++j) {
                    win[0][j] = win[1][j];
                    win[1][j] = win[2][j];
                }
            }
        }
        range_check(hmx);
    }
    // the tile of h (written over G) to global memory: the async proxy reads it
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    if (tid == 0 && ok) {
        tma_store_4d(&A.mh, sbase + L::g, c0, x0, y0, b);
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");   // smem stays valid until read
    }
}

}  // namespace sw
}  // namespace gtr
