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
// Kernels:
//   * gla_fwd_span.cuh (the default): each sequence is cut into spans of chunks that
//     run on separate SMs with purely local state chains; one aggregate per span through
//     a workspace, a look-back fold, and a deferred correction of the later spans'
//     outputs.  Chunk rows are staged with 16-byte cp.async (the scan direction applied
//     only in the row addresses).  An instance that reads z forms the gate from its
//     pre-activation while gating (gtr_gla_fwd_z).
//   * gla_fwd_pipe.cuh (GTR_KERNEL=pipe): the same span decomposition with TMA tensor
//     copies and warp-specialised roles (gating teams, state group, readout group) on
//     mbarrier hand-offs.
//   Both take 64 key channels and 64 value columns per launch: dk = 128 is two launches
//   over the two key halves (the recurrence is separable by key channel; the second
//   adds its output to the first's), dv = 128 two launches over the two value halves
//   (separable by value column; disjoint outputs).
//   Per chunk, in both: gated operands whose decay factors fed to the tensor cores stay
//   inside fp16 (a fast path for chunk decays >= e^-6, a 16-token sub-block path with an
//   exact fp32 diagonal fallback otherwise), then tcgen05.mma (fp16 x fp16 -> fp32 in
//   tensor memory) for dS = K~^T V, the causal scores Qint K~^T and O = Qint S_prev + P V.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/gtr_gla.h"
#include "../../include/gtr_swiglu.h"
#include "sm100_ptx.cuh"

namespace gtr {

using namespace ptx;

constexpr int kChunk = 64;
constexpr int kDV = 64;
constexpr int kSub = 16;              // sub-block length for the decay factorisation
constexpr int kTile = 64 * 128;       // one [64 rows][64 fp16] 128B-swizzled tile
constexpr int kMaxCluster = 16;
constexpr float kDiagMinTotal = 3.3546262e-4f;  // exp(-8): smallest safe sub-block total
constexpr float kFastMinDecay = 2.4787522e-3f;  // exp(-6): smallest chunk decay for the fast path
constexpr float kFastMaxK = 100.f;              // |k| / P stays inside fp16 on the fast path
constexpr float kDiagMaxQ = 20.f;               // |q| / T stays inside fp16 on a diagonal block
constexpr uint64_t kWaitLimitNs = 200ull * 1000ull * 1000ull;  // 200 ms per bounded wait

enum : unsigned { kErrTimeout = 1u, kErrRange = 2u };
constexpr float kHalfMax = 65504.f;   // largest finite fp16

__device__ unsigned int g_error_word;

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
    int dk;        // key channels (the state has dk rows)
    int ldk;       // elements per q / k / g row (dk, or 128 for one half of a dk = 128 call)
    int sstride;   // floats per sequence of init_state / final_state (dk * dv)
    int acc;       // 1: add to the output tile instead of storing it (second key half)
    int ldv;       // elements per v / out row, and floats per state row (dv of the call)
    int vsplit;    // 1: one 64-column value half of a dv = 128 call
};

__device__ __forceinline__ void set_error(unsigned e) { atomicOr(&g_error_word, e); }
// A value about to become an fp16 operand or output must be finite and below 65504
// (a NaN fails the comparison too): else the call reports GTR_ERR_RANGE.
__device__ __forceinline__ void range_check(float mx) {
    if (!(mx <= kHalfMax)) set_error(kErrRange);
}
__device__ __forceinline__ float absmax4(float4 v) {
    return fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
}

// Log-decay of the key-side forget gate from its pre-activation z (GTR news article,
// section "线性注意力到底在省什么"): g = log(sigmoid(z)) / tau = (min(z, 0) - log(1 + e^-|z|))
// / tau, with CUDA's exp / log intrinsics (relative error ~2^-21, far below the fp16
// rounding of z itself; for |z| > 17 the log term falls below fp32's resolution of 1 + x,
// an absolute error under 1e-7 / tau).
__device__ __forceinline__ float gate_of(float z, float inv_tau) {
    return (fminf(z, 0.f) - __logf(1.f + __expf(-fabsf(z)))) * inv_tau;
}
// The log-decay from a staged gate value: g itself, or formed from z (kZ).
template <bool kZ>
__device__ __forceinline__ float2 gate2(float2 x, float inv_tau) {
    if constexpr (kZ) return make_float2(gate_of(x.x, inv_tau), gate_of(x.y, inv_tau));
    return x;
}
template <bool kZ>
__device__ __forceinline__ float gate1(float x, float inv_tau) {
    if constexpr (kZ) return gate_of(x, inv_tau);
    return x;
}

__device__ __forceinline__ float2 ld_h2(const uint8_t *p) {
    return __half22float2(*reinterpret_cast<const __half2 *>(p));
}
__device__ __forceinline__ void st_h2(uint8_t *p, float x, float y) {
    *reinterpret_cast<__half2 *>(p) = __floats2half2_rn(x, y);
}
__device__ __forceinline__ float exp_f(float x) { return __expf(x); }

// 16 TMEM lanes x 256 bit, 4 repeats (32 columns): thread t gets, for repeat c,
// rows (lane base + t/4, + 8) and columns (col + 8c + 2(t%4), +1).
__device__ __forceinline__ void tmem_ld_16x256b_x4(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x4.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

}  // namespace gtr

#include "gla_fwd_span.cuh"
#include "gla_fwd_pipe.cuh"
#include "swiglu_gate.cuh"

namespace gtr {

// ------------------------------------------------------------------ host
}  // namespace gtr

// the backward pass: its kernels, then (below) its C entry points
#include "../../include/gtr_gla_bwd.h"
#include "gla_bwd.cuh"

namespace gtr {
enum KernelKind { kSpan = 0, kSpanShort = 1, kSpanZ = 2, kSpanShortZ = 3, kPipe = 4, kPipeZ = 5, kKinds = 6 };

// the span kernel with two loader warps (kSpan) or four (kSpanShort: short spans),
// reading g or (the Z kinds) its pre-activation z
static bool is_span(int kind) { return kind >= kSpan && kind <= kSpanShortZ; }
// the TMA-staged warp-specialised kernel (g, or its pre-activation z)
static bool is_pipe(int kind) { return kind == kPipe || kind == kPipeZ; }

// A kernel variant: entry point, block size, dynamic shared memory, cache slot.
struct KSpec {
    const void *fn;
    int threads;
    int smem;
    int slot;
};

struct Plan {
    int kind;
    int cluster;       // CTAs working on one sequence (cluster size or spans)
    int clusters;      // groups of such CTAs in the grid
    int span_len;      // chunks per span (span kernel)
    int smem, threads;
    size_t ws_bytes;   // workspace the launch needs (span kernel with >= 2 spans)
};

// The span kernel by default; GTR_KERNEL=pipe (tuning knob) selects the TMA-staged one.
static KSpec spec_of(int kind) {
    switch (kind) {
    case kSpanShort:
        return KSpec{reinterpret_cast<const void *>(&sp::gla_fwd_span_kernel<4, false>), sp::span_threads<4>(),
                     sp::L::alloc, kSpanShort};
    case kSpanZ:
        return KSpec{reinterpret_cast<const void *>(&sp::gla_fwd_span_kernel<2, true>), sp::span_threads<2>(),
                     sp::L::alloc, kSpanZ};
    case kSpanShortZ:
        return KSpec{reinterpret_cast<const void *>(&sp::gla_fwd_span_kernel<4, true>), sp::span_threads<4>(),
                     sp::L::alloc, kSpanShortZ};
    case kPipe:
        return KSpec{reinterpret_cast<const void *>(&pp::gla_fwd_pipe_kernel<false>), pp::kThreads, pp::L::alloc, kPipe};
    case kPipeZ:
        return KSpec{reinterpret_cast<const void *>(&pp::gla_fwd_pipe_kernel<true>), pp::kThreads, pp::L::alloc, kPipeZ};
    default:
        return KSpec{reinterpret_cast<const void *>(&sp::gla_fwd_span_kernel<2, false>), sp::span_threads<2>(),
                     sp::L::alloc, kSpan};
    }
}

static int kind_for(bool gate_z) {
    const char *e = getenv("GTR_KERNEL");
    if (e && !strcmp(e, "pipe")) return gate_z ? kPipeZ : kPipe;
    return gate_z ? kSpanZ : kSpan;
}

static std::mutex g_mu;
static int g_num_sms[64];
// co-resident CTAs of the span kernel per device; 0 = not queried
static int g_span_capacity[64];

static int current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    return dev;
}

static int num_sms(int dev) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_num_sms[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = 148;
        }
        g_num_sms[dev] = n;
    }
    return g_num_sms[dev];
}

static cudaError_t prepare_kernel(const KSpec &k) {
    return cudaFuncSetAttribute(k.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, k.smem);
}

static void fill_config(cudaLaunchConfig_t &cfg, cudaLaunchAttribute *attr, const KSpec &k,
                        int cluster, int clusters, cudaStream_t stream) {
    cfg = cudaLaunchConfig_t{};
    cfg.gridDim = dim3((unsigned)(cluster * clusters), 1, 1);
    cfg.blockDim = dim3((unsigned)k.threads, 1, 1);
    cfg.dynamicSmemBytes = (size_t)k.smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    // all spans of a sequence must be resident together: cooperative launch; the next
    // launch on the stream may start its set-up while this one drains (the kernel waits
    // for its predecessor before touching global memory)
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.numAttrs = 2;
}


static int span_capacity(int dev, int sms, bool query) {
    if (!query) return sms;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (g_span_capacity[dev] != 0) return g_span_capacity[dev];
    }
    const KSpec k = spec_of(kSpan);
    int per_sm = 0;
    if (prepare_kernel(k) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k.fn, k.threads, (size_t)k.smem) != cudaSuccess)
        per_sm = 0;
    cudaGetLastError();
    const int cap = per_sm > 0 ? per_sm * sms : -1;
    std::lock_guard<std::mutex> lk(g_mu);
    g_span_capacity[dev] = cap;
    return cap;
}

// GTR_CLUSTER_SIZE=<n> (tuning knob) forces the cluster size / span count when feasible.
static int forced_cluster() {
    const char *e = getenv("GTR_CLUSTER_SIZE");
    if (!e || !*e) return 0;
    const int n = atoi(e);
    return (n >= 1 && n <= kMaxCluster) ? n : 0;
}

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace of the span kernel: the publish flags of up to 2 * capacity (sequence,
// span) pairs, zero between launches, then the aggregates.  The flags sit at the same
// offset for every shape on a device.
static size_t span_flags_bytes(int cap) {
    return align256((size_t)2 * cap * sp::kFlagStride * sizeof(unsigned));
}
static size_t span_ws_bytes(long n_seq, int spans, int cap) {
    if (spans < 2) return 0;
    return span_flags_bytes(cap) + align256((size_t)n_seq * spans * sp::kAggFloats * sizeof(float));
}

// Span plan: P spans of Lc chunks per sequence (Lc <= 64 when P > 1), grid of whole
// span groups within the co-resident capacity.  Minimises (sequence passes) x
// (chunks per span + 2), the 2 standing for the look-back and the corrections;
// several spans per sequence only while the sequences alone leave SMs idle.
static Plan span_plan(long n_seq, long n_chunks, int cap, int kind, size_t ws_limit) {
    const KSpec k = spec_of(kind);
    Plan best{kind, 1, 1, (int)n_chunks, k.smem, k.threads, 0};
    long best_cost = -1;
    const int fc = forced_cluster();
    for (int P = 1; P <= kMaxCluster && P <= n_chunks && P <= cap; ++P) {
        const long Lc = (n_chunks + P - 1) / P;
        if ((n_chunks + Lc - 1) / Lc != P) continue;   // same split as a smaller P
        if (P > 1 && (Lc > sp::kMaxSpan || n_seq * P > 2L * cap)) continue;
        if (span_ws_bytes(n_seq, P, cap) > ws_limit) continue;   // (P = 1 needs none)
        if (fc > 0 && P != fc) continue;
        const long groups = n_seq < cap / P ? n_seq : cap / P;
        const long passes = (n_seq + groups - 1) / groups;
        const long cost = passes * (Lc + (P > 1 ? 2 : 0));
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best.cluster = P;
            best.clusters = (int)groups;
            best.span_len = (int)Lc;
        }
    }
    if (best_cost < 0 && fc > 0) {   // forced span count not feasible: plan freely
        Plan p1{kind, 1, (int)(n_seq < cap ? n_seq : cap), (int)n_chunks, k.smem, k.threads, 0};
        return p1;
    }
    best.ws_bytes = span_ws_bytes(n_seq, best.cluster, cap);
    if ((kind == kSpan || kind == kSpanZ) && best.cluster > 1 && best.span_len <= sp::kShortSpan) {
        // latency-bound: four loaders
        const KSpec ks = spec_of(kind == kSpan ? kSpanShort : kSpanShortZ);
        best.kind = ks.slot;
        best.threads = ks.threads;
        best.smem = ks.smem;
    }
    return best;
}

// Cluster plan: the cluster size that minimises (waves of clusters) x (rounds per
// sequence + 1), preferring the smaller cluster on ties.

// ws_limit: the largest workspace the caller can provide (the static scratch's size
// for gtr_gla_fwd_static; unlimited otherwise).
static Plan make_plan(long n_seq, long n_chunks, int dk, bool query, size_t ws_limit = ~size_t(0),
                      bool gate_z = false) {
    (void)dk;
    const int kind = kind_for(gate_z);
    const int dev = current_device();
    const int sms = num_sms(dev);
    if (n_chunks == 0) return Plan{kind, 1, 1, 0, 0, 0, 0};   // no launch: the state copy only
    const int cap = span_capacity(dev, sms, query);
    if (cap > 0) return span_plan(n_seq, n_chunks, cap, kind, ws_limit);
    return Plan{-1, 1, 1, 0, 0, 0, 0};   // no co-resident span plan on this device
}

// Library-cached workspace of gtr_gla_fwd, one per device: sized for the largest
// span plan (n_seq * spans <= 2 * capacity), allocated and zero-filled, in the order of
// the caller's stream, by the first call that needs it (or by gtr_gla_init).
struct DefaultWs {
    void *ptr;
    size_t bytes;
};
static DefaultWs g_default_ws[64];

static size_t default_ws_bytes(int cap) {
    if (cap <= 0) return 0;
    return span_flags_bytes(cap) + align256((size_t)2 * cap * sp::kAggFloats * sizeof(float));
}

static cudaError_t default_workspace(int dev, size_t need, cudaStream_t stream, void **ptr) {
    std::lock_guard<std::mutex> lk(g_mu);
    DefaultWs &w = g_default_ws[dev];
    if (w.ptr != nullptr && w.bytes >= need) {
        *ptr = w.ptr;
        return cudaSuccess;
    }
    if (w.ptr != nullptr) return cudaErrorInvalidValue;   // the plan bound guarantees this never happens
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(stream, &cs);
    if (e != cudaSuccess) return e;
    if (cs != cudaStreamCaptureStatusNone) return cudaErrorStreamCaptureUnsupported;
    const int sms = g_num_sms[dev] > 0 ? g_num_sms[dev] : 148;
    const int cap = g_span_capacity[dev] > 0 ? g_span_capacity[dev] : sms;
    size_t bytes = default_ws_bytes(cap);
    if (bytes < need) bytes = need;
    // stream-ordered: the allocation and the zero fill run on the caller's stream ahead
    // of the launch that needs them; the host does not wait
    void *p = nullptr;
    e = cudaMallocAsync(&p, bytes, stream);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(p, 0, bytes, stream);
    if (e != cudaSuccess) {
        cudaFreeAsync(p, stream);
        return e;
    }
    w.ptr = p;
    w.bytes = bytes;
    *ptr = p;
    return cudaSuccess;
}

static thread_local cudaError_t g_last_cuda_error = cudaSuccess;

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ------------------------------------------------------------------ TMA maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
static EncodeTiledFn g_encode = nullptr;

static cudaError_t tensor_map_encoder(EncodeTiledFn *fn) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_encode == nullptr) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        const cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
        if (e != cudaSuccess) return e;
        if (q != cudaDriverEntryPointSuccess || p == nullptr) return cudaErrorNotSupported;
        g_encode = reinterpret_cast<EncodeTiledFn>(p);
    }
    *fn = g_encode;
    return cudaSuccess;
}

// Box heights (bit h: 2^h rows) that the memory-contiguous runs of the chunks of a grid
// scanned in `dir` decompose into: L->R reads whole 64-row boxes; R->L runs end at grid
// rows, T->B and B->T at grid columns, every run also at chunk boundaries.
static unsigned used_heights(int H, int W, int dir) {
    if (dir == GTR_L2R) return 1u << 6;
    const long N = (long)H * W, run = dir == GTR_R2L ? W : H;
    unsigned m = 0;
    for (long p0 = 0; p0 < N; p0 += kChunk) {
        const long pend = p0 + kChunk < N ? p0 + kChunk : N;
        for (long p = p0; p < pend;) {
            const long q = (p / run + 1) * run < pend ? (p / run + 1) * run : pend;
            m |= (unsigned)(q - p);
            p = q;
        }
    }
    return m & 0x7fu;
}

// One tensor ([B, N, heads, pitch] fp16, channels 0 .. d-1 of each row at `ptr`) as a
// row view (d, heads, N, B) or a column view (d, heads, W, H, B), box d x 1 x 2^h rows.
static CUresult encode_map(EncodeTiledFn enc, CUtensorMap *m, const void *ptr, int B, int heads, int H, int W,
                           int d, int pitch, bool column, int h) {
    const cuuint64_t es = 2;
    cuuint64_t dims[5], strides[4];
    cuuint32_t box[5], estr[5] = {1, 1, 1, 1, 1};
    const cuuint64_t N = (cuuint64_t)H * W;
    dims[0] = (cuuint64_t)d;
    dims[1] = (cuuint64_t)heads;
    strides[0] = (cuuint64_t)pitch * es;
    strides[1] = (cuuint64_t)heads * pitch * es;
    box[0] = (cuuint32_t)d;
    box[1] = 1;
    cuuint32_t rank;
    if (!column) {
        rank = 4;
        dims[2] = N;
        dims[3] = (cuuint64_t)B;
        strides[2] = N * heads * pitch * es;
        box[2] = 1u << h;
        box[3] = 1;
    } else {
        rank = 5;
        dims[2] = (cuuint64_t)W;
        dims[3] = (cuuint64_t)H;
        dims[4] = (cuuint64_t)B;
        strides[2] = (cuuint64_t)W * heads * pitch * es;
        strides[3] = N * heads * pitch * es;
        box[2] = 1;
        box[3] = 1u << h;
        box[4] = 1;
    }
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, rank, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

// Encoded maps of the last few (tensors, shape, direction) combinations.
struct MapEntry {
    const void *ptr[4];
    int B, heads, H, W, dir, dev, ldk, ldv;
    unsigned used;
    bool valid;
    pp::Maps maps;
};
static MapEntry g_maps[32];
static int g_maps_next;

static cudaError_t pipe_maps(const Params &prm, int dev, pp::Maps *maps, unsigned *used) {
    const void *ptr[4] = {prm.q, prm.k, prm.g, prm.v};
    {
        std::lock_guard<std::mutex> lk(g_mu);
        for (const MapEntry &m : g_maps) {
            if (m.valid && m.dev == dev && m.B == prm.B && m.heads == prm.heads && m.H == prm.H && m.W == prm.W &&
                m.dir == prm.dir && m.ldk == prm.ldk && m.ldv == prm.ldv && !memcmp(m.ptr, ptr, sizeof(ptr))) {
                *maps = m.maps;
                *used = m.used;
                return cudaSuccess;
            }
        }
    }
    EncodeTiledFn enc = nullptr;
    cudaError_t e = tensor_map_encoder(&enc);
    if (e != cudaSuccess) return e;
    MapEntry ent{};
    memcpy(ent.ptr, ptr, sizeof(ptr));
    ent.B = prm.B;
    ent.heads = prm.heads;
    ent.H = prm.H;
    ent.W = prm.W;
    ent.dir = prm.dir;
    ent.dev = dev;
    ent.ldk = prm.ldk;
    ent.ldv = prm.ldv;
    ent.used = used_heights(prm.H, prm.W, prm.dir);
    const bool column = prm.dir == GTR_T2B || prm.dir == GTR_B2T;
    for (int ten = 0; ten < 4; ++ten)
        for (int h = 0; h < 7; ++h) {
            if (!((ent.used >> h) & 1u)) continue;
            if (encode_map(enc, &ent.maps.m[ten][h], ptr[ten], prm.B, prm.heads, prm.H, prm.W,
                           ten == 3 ? kDV : pp::kDK, ten == 3 ? prm.ldv : prm.ldk, column, h) != CUDA_SUCCESS)
                return cudaErrorInvalidValue;
        }
    ent.valid = true;
    std::lock_guard<std::mutex> lk(g_mu);
    g_maps[g_maps_next] = ent;
    g_maps_next = (g_maps_next + 1) % (int)(sizeof(g_maps) / sizeof(g_maps[0]));
    *maps = ent.maps;
    *used = ent.used;
    return cudaSuccess;
}

static cudaError_t launch(const Params &prm, const Plan &pl, void *workspace, cudaStream_t stream,
                          float inv_tau = 1.f) {
    const int dev = current_device();
    if (prm.n_chunks == 0) {
        // an empty grid: the final state is the initial one (zero without one), in the
        // order of the caller's stream
        if (prm.sf == nullptr) return cudaSuccess;
        const size_t bytes = (size_t)prm.n_seq * prm.sstride * sizeof(float);
        return prm.s0 != nullptr ? cudaMemcpyAsync(prm.sf, prm.s0, bytes, cudaMemcpyDeviceToDevice, stream)
                                 : cudaMemsetAsync(prm.sf, 0, bytes, stream);
    }
    if (pl.kind < 0) return cudaErrorNotSupported;
    const KSpec k = spec_of(pl.kind);
    cudaError_t e = prepare_kernel(k);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr[2];
    fill_config(cfg, attr, k, pl.cluster, pl.clusters, stream);
    if (prm.ldv == 2 * kDV && !prm.vsplit) {
        // dv = 128: the recurrence is separable by value column too (column j of the
        // state sees only v_j), so the two 64-column halves are independent calls that
        // write disjoint output columns and state columns
        for (int half = 0; half < 2; ++half) {
            Params ph = prm;
            const size_t co = (size_t)half * kDV;
            ph.v = prm.v + co;
            ph.out = prm.out + co;
            if (prm.s0 != nullptr) ph.s0 = prm.s0 + co;
            if (prm.sf != nullptr) ph.sf = prm.sf + co;
            ph.vsplit = 1;
            e = launch(ph, pl, workspace, stream, inv_tau);
            if (e != cudaSuccess) return e;
        }
        return cudaSuccess;
    }
    if (prm.dk == 2 * pp::kDK) {
        // dk = 128: the recurrence is separable by key channel (row i of the state sees
        // only channel i of k and of the decay), and the output sums the two halves'
        // contributions: channels 0..63 (state rows 0..63) store the output, channels
        // 64..127 (state rows 64..127) add to it, in stream order
        for (int half = 0; half < 2; ++half) {
            Params ph = prm;
            const size_t co = (size_t)half * pp::kDK;
            ph.q = prm.q + co;
            ph.k = prm.k + co;
            ph.g = prm.g + co;
            ph.ldk = prm.dk;
            ph.dk = pp::kDK;
            if (prm.s0 != nullptr) ph.s0 = prm.s0 + co * prm.ldv;
            if (prm.sf != nullptr) ph.sf = prm.sf + co * prm.ldv;
            ph.acc = half;
            e = launch(ph, pl, workspace, stream, inv_tau);
            if (e != cudaSuccess) return e;
        }
        return cudaSuccess;
    }
    if (is_pipe(pl.kind)) {
        static thread_local pp::Args a;
        a = pp::Args{};
        e = pipe_maps(prm, dev, &a.maps, &a.used);
        if (e != cudaSuccess) return e;
        a.P = prm;
        a.PS = pl.cluster;
        a.Lc = pl.span_len;
        a.inv_tau = inv_tau;
        if (pl.ws_bytes > 0) {
            uint8_t *base = static_cast<uint8_t *>(workspace);
            const int cap = span_capacity(dev, num_sms(dev), true);
            a.flags = reinterpret_cast<unsigned *>(base);
            a.ws = reinterpret_cast<float *>(base + span_flags_bytes(cap));
        }
        void *args[] = {&a};
        return cudaLaunchKernelExC(&cfg, k.fn, args);
    }
    if (is_span(pl.kind)) {
        sp::Work wk{};
        wk.inv_tau = inv_tau;
        wk.P = pl.cluster;
        wk.Lc = pl.span_len;
        if (pl.ws_bytes > 0) {
            uint8_t *base = static_cast<uint8_t *>(workspace);
            const int cap = span_capacity(dev, num_sms(dev), true);
            wk.flags = reinterpret_cast<unsigned *>(base);
            wk.ws = reinterpret_cast<float *>(base + span_flags_bytes(cap));
        }
        void *args[] = {const_cast<Params *>(&prm), &wk};
        return cudaLaunchKernelExC(&cfg, k.fn, args);
    }
    void *args[] = {const_cast<Params *>(&prm)};
    return cudaLaunchKernelExC(&cfg, k.fn, args);
}

}  // namespace gtr

using namespace gtr;

#include <nvtx3/nvToolsExt.h>

// An NVTX range over a library call (a no-op unless a profiler is attached): the
// calls, the stack's recording and the SwiGLU launch show up on a timeline.
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

static gtr_status_t check_args(const void *q, const void *k, const void *v, const void *g,
                               int B, int heads, int H, int W, int dk, int dv, int dir,
                               int chunk, const float *s0, const void *out, const float *sf) {
    if (B <= 0 || heads <= 0 || H < 0 || W < 0 || dk <= 0 || dv <= 0) return GTR_ERR_INVALID_ARG;
    const bool empty = (long long)H * W == 0;   // an empty grid reads and writes no token
    if (!empty && (!q || !k || !v || !g || !out)) return GTR_ERR_INVALID_ARG;
    if (dir < 0 || dir > 3) return GTR_ERR_INVALID_ARG;
    if (chunk <= 0) return GTR_ERR_INVALID_ARG;
    if (chunk != kChunk) return GTR_ERR_UNSUPPORTED;
    if ((dk != 64 && dk != 128) || (dv != 64 && dv != 128)) return GTR_ERR_UNSUPPORTED;
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

static Params make_params(const gtr_half_t *q, const gtr_half_t *k, const gtr_half_t *v,
                          const gtr_half_t *g, int B, int heads, int Hgrid, int Wgrid, int direction,
                          const float *init_state, gtr_half_t *out, float *final_state, int dk, int dv) {
    Params prm{};
    prm.dk = dk;
    prm.ldk = dk;
    prm.sstride = dk * dv;
    prm.acc = 0;
    prm.ldv = dv;
    prm.vsplit = 0;
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
    return prm;
}

static gtr_status_t cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return GTR_OK;
    g_last_cuda_error = e;
    cudaGetLastError();   // clear a non-sticky error
    return GTR_ERR_CUDA;
}

extern "C" gtr_status_t gtr_gla_fwd(const gtr_half_t *q, const gtr_half_t *k,
                                    const gtr_half_t *v, const gtr_half_t *g, int B, int heads,
                                    int Hgrid, int Wgrid, int dk, int dv, int direction, int chunk,
                                    const float *init_state, gtr_half_t *out, float *final_state,
                                    void *stream) {
    NvtxRange nvtx_range("gtr_gla_fwd");
    const gtr_status_t st = check_args(q, k, v, g, B, heads, Hgrid, Wgrid, dk, dv, direction,
                                       chunk, init_state, out, final_state);
    if (st != GTR_OK) return st;
    const Params prm = make_params(q, k, v, g, B, heads, Hgrid, Wgrid, direction, init_state, out,
                                   final_state, dk, dv);
    const Plan pl = make_plan(prm.n_seq, prm.n_chunks, dk, true);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    void *ws = nullptr;
    if (pl.ws_bytes > 0) {
        const gtr_status_t wst = cuda_status(default_workspace(current_device(), pl.ws_bytes, s, &ws));
        if (wst != GTR_OK) return wst;
    }
    return cuda_status(launch(prm, pl, ws, s));
}

extern "C" gtr_status_t gtr_gla_fwd_z(const gtr_half_t *q, const gtr_half_t *k, const gtr_half_t *v,
                                      const gtr_half_t *z, float tau, int B, int heads, int Hgrid, int Wgrid,
                                      int dk, int dv, int direction, int chunk, const float *init_state,
                                      gtr_half_t *out, float *final_state, void *stream) {
    NvtxRange nvtx_range("gtr_gla_fwd_z");
    const gtr_status_t st = check_args(q, k, v, z, B, heads, Hgrid, Wgrid, dk, dv, direction, chunk, init_state,
                                       out, final_state);
    if (st != GTR_OK) return st;
    if (!(tau > 0.f) || !(tau < 3.0e38f)) return GTR_ERR_INVALID_ARG;
    if ((long long)Hgrid * Wgrid == 0)   // no token: the state copy of the plain call
        return gtr_gla_fwd(q, k, v, z, B, heads, Hgrid, Wgrid, dk, dv, direction, chunk, init_state, out,
                           final_state, stream);
    const Params prm = make_params(q, k, v, z, B, heads, Hgrid, Wgrid, direction, init_state, out, final_state, dk, dv);
    const Plan pl = make_plan(prm.n_seq, prm.n_chunks, dk, true, ~size_t(0), true);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    void *ws = nullptr;
    if (pl.ws_bytes > 0) {
        const gtr_status_t wst = cuda_status(default_workspace(current_device(), pl.ws_bytes, s, &ws));
        if (wst != GTR_OK) return wst;
    }
    return cuda_status(launch(prm, pl, ws, s, 1.f / tau));
}

// ------------------------------------------------------------------ layer stacks
// Graphs of recorded stacks, keyed by the layer list and shape (a few recent ones).
struct StackEntry {
    int dev, n, B, heads, H, W, dk, dv;
    gtr_gla_layer_t layers[64];
    cudaGraphExec_t exec;
};
static StackEntry g_stacks[8];
static int g_stacks_next;

static bool same_layer(const gtr_gla_layer_t &a, const gtr_gla_layer_t &b) {   // field by field (no padding)
    return a.q == b.q && a.k == b.k && a.v == b.v && a.g == b.g && a.init_state == b.init_state && a.out == b.out &&
           a.final_state == b.final_state && a.direction == b.direction;
}

static bool same_stack(const StackEntry &e, int dev, const gtr_gla_layer_t *layers, int n, int B, int heads, int H,
                       int W, int dk, int dv) {
    if (e.exec == nullptr || e.dev != dev || e.n != n || e.B != B || e.heads != heads || e.H != H || e.W != W ||
        e.dk != dk || e.dv != dv)
        return false;
    for (int i = 0; i < n; ++i)
        if (!same_layer(e.layers[i], layers[i])) return false;
    return true;
}

// per device: the private stream that stacks are recorded on
static cudaStream_t g_rec_stream[64];

extern "C" gtr_status_t gtr_gla_fwd_stack(const gtr_gla_layer_t *layers, int n_layers, int B, int heads, int Hgrid,
                                          int Wgrid, int dk, int dv, int chunk, void *stream) {
    NvtxRange nvtx_range("gtr_gla_fwd_stack");
    if (layers == nullptr || n_layers < 1 || n_layers > 64) return GTR_ERR_INVALID_ARG;
    for (int i = 0; i < n_layers; ++i) {
        const gtr_gla_layer_t &L = layers[i];
        const gtr_status_t st = check_args(L.q, L.k, L.v, L.g, B, heads, Hgrid, Wgrid, dk, dv, L.direction, chunk,
                                           L.init_state, L.out, L.final_state);
        if (st != GTR_OK) return st;
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int dev = current_device();
    // every layer has the same plan; its workspace exists before any recording starts
    const Plan pl = make_plan((long)B * heads, (long)(((long long)Hgrid * Wgrid + kChunk - 1) / kChunk), dk, true);
    void *ws = nullptr;
    if (pl.ws_bytes > 0) {
        const gtr_status_t wst = cuda_status(default_workspace(dev, pl.ws_bytes, s, &ws));
        if (wst != GTR_OK) return wst;
    }
    const auto enqueue = [&]() -> cudaError_t {
        for (int i = 0; i < n_layers; ++i) {
            const gtr_gla_layer_t &L = layers[i];
            const Params prm = make_params(L.q, L.k, L.v, L.g, B, heads, Hgrid, Wgrid, L.direction, L.init_state,
                                           L.out, L.final_state, dk, dv);
            const cudaError_t e = launch(prm, pl, ws, s);
            if (e != cudaSuccess) return e;
        }
        return cudaSuccess;
    };
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(s, &cs);
    if (e != cudaSuccess) return cuda_status(e);
    if (cs != cudaStreamCaptureStatusNone || (long long)Hgrid * Wgrid == 0) return cuda_status(enqueue());
    {
        std::lock_guard<std::mutex> lk(g_mu);
        for (const StackEntry &en : g_stacks)
            if (same_stack(en, dev, layers, n_layers, B, heads, Hgrid, Wgrid, dk, dv))
                return cuda_status(cudaGraphLaunch(en.exec, s));
    }
    // record the stack once, then replay it on the caller's stream.  Recording runs on a
    // private stream: the caller's may be the legacy default stream, which cannot be
    // captured (recording executes nothing, so the private stream needs no ordering)
    cudaStream_t rec = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (g_rec_stream[dev] == nullptr &&
            (e = cudaStreamCreateWithFlags(&g_rec_stream[dev], cudaStreamNonBlocking)) != cudaSuccess) {
            g_rec_stream[dev] = nullptr;
            return cuda_status(e);
        }
        rec = g_rec_stream[dev];
    }
    const cudaStream_t caller = s;
    s = rec;   // `enqueue` launches on `s`
    e = cudaStreamBeginCapture(rec, cudaStreamCaptureModeThreadLocal);
    if (e != cudaSuccess) return cuda_status(e);
    const cudaError_t le = enqueue();
    cudaGraph_t graph = nullptr;
    e = cudaStreamEndCapture(rec, &graph);
    s = caller;
    if (le != cudaSuccess || e != cudaSuccess) {
        if (graph) cudaGraphDestroy(graph);
        return cuda_status(le != cudaSuccess ? le : e);
    }
    cudaGraphExec_t exec = nullptr;
    e = cudaGraphInstantiate(&exec, graph, 0);
    cudaGraphDestroy(graph);
    if (e != cudaSuccess) return cuda_status(e);
    e = cudaGraphLaunch(exec, s);
    std::lock_guard<std::mutex> lk(g_mu);
    StackEntry &slot = g_stacks[g_stacks_next];
    if (slot.exec != nullptr) cudaGraphExecDestroy(slot.exec);
    slot.dev = dev;
    slot.n = n_layers;
    slot.B = B;
    slot.heads = heads;
    slot.H = Hgrid;
    slot.W = Wgrid;
    slot.dk = dk;
    slot.dv = dv;
    memcpy(slot.layers, layers, sizeof(gtr_gla_layer_t) * (size_t)n_layers);
    slot.exec = exec;
    g_stacks_next = (g_stacks_next + 1) % (int)(sizeof(g_stacks) / sizeof(g_stacks[0]));
    return cuda_status(e);
}

extern "C" gtr_status_t gtr_gla_init(void *stream) {
    NvtxRange nvtx_range("gtr_gla_init");
    const int dev = current_device();
    const int cap = span_capacity(dev, num_sms(dev), true);
    if (cap <= 0) return GTR_OK;   // no span plan on this device: no workspace
    void *ws = nullptr;
    return cuda_status(default_workspace(dev, default_ws_bytes(cap), reinterpret_cast<cudaStream_t>(stream), &ws));
}

extern "C" size_t gtr_gla_workspace_bytes(int B, int heads, int Hgrid, int Wgrid, int dk, int dv,
                                          int chunk) {
    if (B <= 0 || heads <= 0 || Hgrid < 0 || Wgrid < 0 || chunk != kChunk) return 0;
    if ((dk != 64 && dk != 128) || (dv != 64 && dv != 128)) return 0;
    const long long N = (long long)Hgrid * Wgrid;
    if (N > 0x7fffffffLL || (long long)B * heads > 0x7fffffffLL) return 0;
    int ndev = 0;
    const bool gpu = cudaGetDeviceCount(&ndev) == cudaSuccess && ndev > 0;
    cudaGetLastError();
    return make_plan((long)B * heads, (long)((N + kChunk - 1) / kChunk), dk, gpu).ws_bytes;
}

extern "C" gtr_status_t gtr_gla_fwd_ws(const gtr_half_t *q, const gtr_half_t *k,
                                       const gtr_half_t *v, const gtr_half_t *g, int B, int heads,
                                       int Hgrid, int Wgrid, int dk, int dv, int direction,
                                       int chunk, const float *init_state, gtr_half_t *out,
                                       float *final_state, void *workspace, size_t workspace_bytes,
                                       void *stream) {
    NvtxRange nvtx_range("gtr_gla_fwd_ws");
    const gtr_status_t st = check_args(q, k, v, g, B, heads, Hgrid, Wgrid, dk, dv, direction,
                                       chunk, init_state, out, final_state);
    if (st != GTR_OK) return st;
    const Params prm = make_params(q, k, v, g, B, heads, Hgrid, Wgrid, direction, init_state, out,
                                   final_state, dk, dv);
    const Plan pl = make_plan(prm.n_seq, prm.n_chunks, dk, true);
    if (pl.ws_bytes > 0 &&
        (workspace == nullptr || workspace_bytes < pl.ws_bytes ||
         (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0))
        return GTR_ERR_INVALID_ARG;
    return cuda_status(launch(prm, pl, workspace, reinterpret_cast<cudaStream_t>(stream)));
}

// ------------------------------------------------------------------ static scratch
namespace gtr {

constexpr size_t kStaticWsBytes = GTR_STATIC_WS_BYTES;
static __device__ __align__(256) unsigned char g_static_ws[kStaticWsBytes];
static void *g_static_ws_ptr[64];

// Device address of the static scratch on the current device `dev`, looked up once
// (with `dev` current); the first lookup also zero-fills the publish flags.
static cudaError_t static_scratch(int dev, cudaStream_t stream, void **ptr) {
    const int cap = span_capacity(dev, num_sms(dev), true);
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_static_ws_ptr[dev] == nullptr) {
        // the set-up synchronises the device: not inside a stream capture
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        cudaError_t ce = cudaStreamIsCapturing(stream, &cs);
        if (ce != cudaSuccess) return ce;
        if (cs != cudaStreamCaptureStatusNone) return cudaErrorStreamCaptureUnsupported;
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_static_ws);
        if (e != cudaSuccess) return e;
        e = cudaMemset(p, 0, span_flags_bytes(cap > 0 ? cap : num_sms(dev)));
        if (e == cudaSuccess) e = cudaDeviceSynchronize();
        if (e != cudaSuccess) return e;
        g_static_ws_ptr[dev] = p;
    }
    *ptr = g_static_ws_ptr[dev];
    return cudaSuccess;
}

}  // namespace gtr

extern "C" gtr_status_t gtr_gla_fwd_static(const gtr_half_t *q, const gtr_half_t *k,
                                           const gtr_half_t *v, const gtr_half_t *g, int B,
                                           int heads, int Hgrid, int Wgrid, int dk, int dv,
                                           int direction, int chunk, const float *init_state,
                                           gtr_half_t *out, float *final_state, void *stream) {
    NvtxRange nvtx_range("gtr_gla_fwd_static");
    const gtr_status_t st = check_args(q, k, v, g, B, heads, Hgrid, Wgrid, dk, dv, direction,
                                       chunk, init_state, out, final_state);
    if (st != GTR_OK) return st;
    const Params prm = make_params(q, k, v, g, B, heads, Hgrid, Wgrid, direction, init_state, out,
                                   final_state, dk, dv);
    // the cheapest plan whose workspace fits the scratch (one span per sequence needs none)
    const Plan pl = make_plan(prm.n_seq, prm.n_chunks, dk, true, kStaticWsBytes);
    if (pl.ws_bytes > kStaticWsBytes) return GTR_ERR_UNSUPPORTED;
    void *ws = nullptr;
    if (pl.ws_bytes > 0) {
        const gtr_status_t wst =
            cuda_status(static_scratch(current_device(), reinterpret_cast<cudaStream_t>(stream), &ws));
        if (wst != GTR_OK) return wst;
    }
    return cuda_status(launch(prm, pl, ws, reinterpret_cast<cudaStream_t>(stream)));
}

namespace gtr {

// Self-test of the device-side failure path: thread 0 waits on an mbarrier that
// nothing arrives on and thread 32 polls a flag that nothing sets, each through the
// bounded waits the forward kernels use, for limit_ns; both report kErrTimeout
// through the device error word and the kernel ends normally.
static __device__ unsigned g_selftest_flag;   // never written

__global__ void selftest_wait_kernel(uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t never;
    if (threadIdx.x == 0) {
        mbar_init(&never, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !mbar_wait_bounded(&never, 0, limit_ns)) set_error(kErrTimeout);
    if (threadIdx.x == 32 && !sp::flag_wait_bounded(&g_selftest_flag, limit_ns)) set_error(kErrTimeout);
}

}  // namespace gtr

extern "C" gtr_status_t gtr_gla_selftest_timeout(unsigned limit_us, void *stream) {
    if (limit_us == 0 || limit_us > 1000000u) return GTR_ERR_INVALID_ARG;
    selftest_wait_kernel<<<1, 64, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        (uint64_t)limit_us * 1000ull);
    return cuda_status(cudaGetLastError());
}

extern "C" gtr_status_t gtr_gla_device_status(void *stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) {
        cudaGetLastError();
        return GTR_ERR_CUDA;
    }
    unsigned word = 0;
    if (cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word)) != cudaSuccess) return GTR_ERR_CUDA;
    if (word == kErrRange) {
        const unsigned zero = 0;
        cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero));
        return GTR_ERR_RANGE;
    }
    if (word != 0) {
        const unsigned zero = 0;
        cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero));
        // a span launch that timed out can leave publish flags set: clear the library's
        // workspaces of this device (cached and static) so the next call starts from zero
        const int dev = current_device();
        std::lock_guard<std::mutex> lk(g_mu);
        if (g_default_ws[dev].ptr != nullptr) cudaMemset(g_default_ws[dev].ptr, 0, g_default_ws[dev].bytes);
        if (g_static_ws_ptr[dev] != nullptr) cudaMemset(g_static_ws_ptr[dev], 0, kStaticWsBytes);
        cudaDeviceSynchronize();
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
    case GTR_ERR_RANGE: return "an fp16 operand or output left the fp16 range";
    }
    return "unknown status";
}

extern "C" gtr_status_t gtr_gla_plan(int B, int heads, int Hgrid, int Wgrid, int dk, int dv,
                                     int *cluster_size, int *num_clusters, int *smem_bytes) {
    if (B <= 0 || heads <= 0 || Hgrid < 0 || Wgrid < 0) return GTR_ERR_INVALID_ARG;
    if ((dk != 64 && dk != 128) || (dv != 64 && dv != 128)) return GTR_ERR_UNSUPPORTED;
    const long long N = (long long)Hgrid * Wgrid;
    int ndev = 0;
    const bool gpu = cudaGetDeviceCount(&ndev) == cudaSuccess && ndev > 0;
    cudaGetLastError();
    const Plan pl = make_plan((long)B * heads, (long)((N + kChunk - 1) / kChunk), dk, gpu);
    if (cluster_size) *cluster_size = pl.cluster;
    if (num_clusters) *num_clusters = pl.clusters;
    if (smem_bytes) *smem_bytes = pl.smem;
    return GTR_OK;
}

namespace gtr {

// ------------------------------------------------------------------ backward
// Workspace of one key half: U -> h_c and W -> dh_{c+1} tiles, chunk log-decays and
// x totals, the per-sequence constants.
struct BwdWs {
    size_t hs, dhs, bc, xc, cst, bytes;
};
static BwdWs bwd_ws_layout(long n_seq, long nc) {
    BwdWs w{};
    const size_t tiles = align256((size_t)n_seq * nc * 4096 * sizeof(float));
    const size_t vecs = align256((size_t)n_seq * nc * bw::kC * sizeof(float));
    w.hs = 0;
    w.dhs = w.hs + tiles;
    w.bc = w.dhs + tiles;
    w.xc = w.bc + vecs;
    w.cst = w.xc + vecs;
    w.bytes = w.cst + align256((size_t)n_seq * bw::kC * sizeof(float));
    return w;
}

static gtr_status_t check_bwd_args(const void *q, const void *k, const void *v, const void *g, const void *dout,
                                   const float *s0, const float *dsf, int B, int heads, int H, int W, int dk,
                                   int dv, int dir, int chunk, const float *gq, const float *gk, const float *gv,
                                   const float *gg, const float *gs0) {
    if (B <= 0 || heads <= 0 || H < 0 || W < 0 || dk <= 0 || dv <= 0) return GTR_ERR_INVALID_ARG;
    if (dir < 0 || dir > 3 || chunk <= 0) return GTR_ERR_INVALID_ARG;
    if (chunk != kChunk || (dk != 64 && dk != 128) || dv != 64) return GTR_ERR_UNSUPPORTED;
    const long long N = (long long)H * W;
    const long long rows = (long long)B * N * heads;
    if (N > 0x7fffffffLL || rows * (long long)dk > 0x7fffffffLL || rows * dv > 0x7fffffffLL)
        return GTR_ERR_INVALID_ARG;
    const bool empty = N == 0;
    const void *need[] = {q, k, v, g, dout, gq, gk, gv, gg};
    for (const void *p : need)
        if (!empty && (!p || !aligned16(p))) return GTR_ERR_INVALID_ARG;
    const void *opt[] = {s0, dsf, gs0};
    for (const void *p : opt)
        if (p && !aligned16(p)) return GTR_ERR_INVALID_ARG;
    const long long hk = rows * dk * 2, hv = rows * dv * 2, fk = rows * dk * 4, fv = rows * dv * 4;
    const long long st = (long long)B * heads * dk * dv * 4;
    struct Span {
        const void *p;
        long long n;
    };
    const Span ins[] = {{q, hk}, {k, hk}, {v, hv}, {g, hk}, {dout, hv}, {s0, st}, {dsf, st}};
    const Span outs[] = {{gq, fk}, {gk, fk}, {gv, fv}, {gg, fk}, {gs0, st}};
    auto overlap = [](const Span &a, const Span &b) {
        const uintptr_t x = reinterpret_cast<uintptr_t>(a.p), y = reinterpret_cast<uintptr_t>(b.p);
        return a.p && b.p && a.n > 0 && b.n > 0 && x < y + (uintptr_t)b.n && y < x + (uintptr_t)a.n;
    };
    for (int i = 0; i < 5; ++i) {
        if (empty && i < 4) continue;
        for (const Span &in : ins)
            if (overlap(outs[i], in)) return GTR_ERR_INVALID_ARG;
        for (int j = i + 1; j < 5; ++j)
            if (!(empty && j < 4) && overlap(outs[i], outs[j])) return GTR_ERR_INVALID_ARG;
    }
    return GTR_OK;
}

static cudaError_t bwd_launch(const bw::Args &a, cudaStream_t stream) {
    const size_t smem1 = bw::kLocalSmem;
    cudaError_t e = cudaFuncSetAttribute(bw::gla_bwd_local_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem1);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(bw::gla_bwd_grad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)bw::kGradSmem);
    if (e != cudaSuccess) return e;
    const unsigned chunks = (unsigned)((long)a.n_seq * a.nc);
    bw::gla_bwd_local_kernel<<<chunks, bw::kThreads, smem1, stream>>>(a);
    bw::gla_bwd_scan_kernel<<<(unsigned)a.n_seq * 16u, bw::kThreads, 0, stream>>>(a);
    bw::gla_bwd_grad_kernel<<<chunks, bw::kThreads, bw::kGradSmem, stream>>>(a);
    bw::gla_bwd_dg_kernel<<<chunks, bw::kThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace gtr

extern "C" size_t gtr_gla_bwd_workspace_bytes(int B, int heads, int Hgrid, int Wgrid, int dk, int dv,
                                              int chunk) {
    using namespace gtr;
    if (B <= 0 || heads <= 0 || Hgrid < 0 || Wgrid < 0 || chunk != kChunk || (dk != 64 && dk != 128) || dv != 64)
        return 0;
    const long long N = (long long)Hgrid * Wgrid;
    if (N == 0 || N > 0x7fffffffLL || (long long)B * N * heads * dk > 0x7fffffffLL) return 0;
    return bwd_ws_layout((long)B * heads, (long)((N + kChunk - 1) / kChunk)).bytes;
}

extern "C" gtr_status_t gtr_gla_bwd(const gtr_half_t *q, const gtr_half_t *k, const gtr_half_t *v,
                                    const gtr_half_t *g, const gtr_half_t *d_out, const float *init_state,
                                    const float *d_final_state, int B, int heads, int Hgrid, int Wgrid,
                                    int dk, int dv, int direction, int chunk, float *grad_q, float *grad_k,
                                    float *grad_v, float *grad_g, float *grad_init_state, void *workspace,
                                    size_t workspace_bytes, void *stream) {
    using namespace gtr;
    NvtxRange nvtx_range("gtr_gla_bwd");
    gtr_status_t st = check_bwd_args(q, k, v, g, d_out, init_state, d_final_state, B, heads, Hgrid, Wgrid, dk,
                                     dv, direction, chunk, grad_q, grad_k, grad_v, grad_g, grad_init_state);
    if (st != GTR_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const long long N = (long long)Hgrid * Wgrid;
    const long n_seq = (long)B * heads;
    const size_t st_bytes = (size_t)n_seq * dk * dv * sizeof(float);
    if (N == 0) {   // no position: dL/dS0 = dL/dS_final
        if (grad_init_state == nullptr) return GTR_OK;
        return cuda_status(d_final_state ? cudaMemcpyAsync(grad_init_state, d_final_state, st_bytes,
                                                           cudaMemcpyDeviceToDevice, s)
                                         : cudaMemsetAsync(grad_init_state, 0, st_bytes, s));
    }
    const long nc = (long)((N + kChunk - 1) / kChunk);
    const BwdWs lay = bwd_ws_layout(n_seq, nc);
    if (workspace == nullptr || workspace_bytes < lay.bytes || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return GTR_ERR_INVALID_ARG;
    {   // the workspace may not overlap any tensor of the call
        const long long rows = (long long)B * N * heads, st = (long long)n_seq * dk * dv * 4;
        const void *ps[] = {q, k, v, g, d_out, init_state, d_final_state, grad_q, grad_k, grad_v, grad_g,
                            grad_init_state};
        const long long ns[] = {rows * dk * 2, rows * dk * 2, rows * dv * 2, rows * dk * 2, rows * dv * 2, st, st,
                                rows * dk * 4, rows * dk * 4, rows * dv * 4, rows * dk * 4, st};
        const uintptr_t w0 = reinterpret_cast<uintptr_t>(workspace), w1 = w0 + lay.bytes;
        for (int i = 0; i < 12; ++i) {
            const uintptr_t p0 = reinterpret_cast<uintptr_t>(ps[i]);
            if (ps[i] != nullptr && p0 < w1 && w0 < p0 + (uintptr_t)ns[i]) return GTR_ERR_INVALID_ARG;
        }
    }
    uint8_t *wb = static_cast<uint8_t *>(workspace);
    for (int half = 0; half < dk / 64; ++half) {
        bw::Args a{};
        const size_t ko = (size_t)half * 64;
        a.q = reinterpret_cast<const __half *>(q) + ko;
        a.k = reinterpret_cast<const __half *>(k) + ko;
        a.g = reinterpret_cast<const __half *>(g) + ko;
        a.v = reinterpret_cast<const __half *>(v);
        a.dout = reinterpret_cast<const __half *>(d_out);
        a.s0 = init_state ? init_state + ko * dv : nullptr;
        a.dsf = d_final_state ? d_final_state + ko * dv : nullptr;
        a.dq = grad_q + ko;
        a.dk = grad_k + ko;
        a.dg = grad_g + ko;
        a.dv = grad_v;
        a.ds0 = grad_init_state ? grad_init_state + ko * dv : nullptr;
        a.hs = reinterpret_cast<float *>(wb + lay.hs);
        a.dhs = reinterpret_cast<float *>(wb + lay.dhs);
        a.bc = reinterpret_cast<float *>(wb + lay.bc);
        a.xc = reinterpret_cast<float *>(wb + lay.xc);
        a.cst = reinterpret_cast<float *>(wb + lay.cst);
        a.heads = heads;
        a.H = Hgrid;
        a.W = Wgrid;
        a.N = (int)N;
        a.dir = direction;
        a.n_seq = (int)n_seq;
        a.nc = (int)nc;
        a.ldk = dk;
        a.sstride = dk * dv;
        a.acc_dv = half;
        st = cuda_status(bwd_launch(a, s));
        if (st != GTR_OK) return st;
    }
    return GTR_OK;
}


extern "C" const char *gtr_gla_version(void) { return "0.3.0"; }

extern "C" const char *gtr_gla_last_error(void) {
    return g_last_cuda_error == cudaSuccess ? "no error" : cudaGetErrorString(g_last_cuda_error);
}

// ------------------------------------------------------------------ Spatial SwiGLU
namespace gtr {

// One activation tensor ([B, H, W, C] fp16, channels contiguous) as (C, W, H, B),
// box 64 channels x box_w x box_h x 1.
static CUresult encode_act_map(EncodeTiledFn enc, CUtensorMap *m, const void *ptr, int B, int H, int W, int C,
                               int box_w, int box_h) {
    const cuuint64_t es = 2;
    const cuuint64_t dims[4] = {(cuuint64_t)C, (cuuint64_t)W, (cuuint64_t)H, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)C * es, (cuuint64_t)W * C * es, (cuuint64_t)H * W * C * es};
    const cuuint32_t box[4] = {(cuuint32_t)sw::kTC, (cuuint32_t)box_w, (cuuint32_t)box_h, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

struct SwMapEntry {
    const void *g, *u, *h;
    int B, H, W, C, dev;
    bool valid;
    CUtensorMap mu, mg, mh;
};
static SwMapEntry g_swmaps[16];
static int g_swmaps_next;

static cudaError_t swiglu_maps(const void *G, const void *U, const void *h, int B, int H, int W, int C, int dev,
                               sw::Args *a) {
    {
        std::lock_guard<std::mutex> lk(g_mu);
        for (const SwMapEntry &e : g_swmaps)
            if (e.valid && e.g == G && e.u == U && e.h == h && e.B == B && e.H == H && e.W == W && e.C == C &&
                e.dev == dev) {
                a->mu = e.mu;
                a->mg = e.mg;
                a->mh = e.mh;
                return cudaSuccess;
            }
    }
    EncodeTiledFn enc = nullptr;
    const cudaError_t e = tensor_map_encoder(&enc);
    if (e != cudaSuccess) return e;
    SwMapEntry ent{};
    ent.g = G;
    ent.u = U;
    ent.h = h;
    ent.B = B;
    ent.H = H;
    ent.W = W;
    ent.C = C;
    ent.dev = dev;
    if (encode_act_map(enc, &ent.mu, U, B, H, W, C, sw::kTX + 2, sw::kTY + 2) != CUDA_SUCCESS ||
        encode_act_map(enc, &ent.mg, G, B, H, W, C, sw::kTX, sw::kTY) != CUDA_SUCCESS ||
        encode_act_map(enc, &ent.mh, h, B, H, W, C, sw::kTX, sw::kTY) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    ent.valid = true;
    std::lock_guard<std::mutex> lk(g_mu);
    g_swmaps[g_swmaps_next] = ent;
    g_swmaps_next = (g_swmaps_next + 1) % (int)(sizeof(g_swmaps) / sizeof(g_swmaps[0]));
    a->mu = ent.mu;
    a->mg = ent.mg;
    a->mh = ent.mh;
    return cudaSuccess;
}

}  // namespace gtr

extern "C" gtr_status_t gtr_spatial_swiglu_gate(const gtr_half_t *G, const gtr_half_t *U, const float *w,
                                                const float *bias, int B, int H, int W, int C, gtr_half_t *out,
                                                void *stream) {
    NvtxRange nvtx_range("gtr_spatial_swiglu_gate");
    if (B < 0 || H < 0 || W < 0 || C < 0) return GTR_ERR_INVALID_ARG;
    const long long n = (long long)B * H * W * C;
    if (n == 0) return GTR_OK;   // nothing to read or write
    if (!G || !U || !w || !out) return GTR_ERR_INVALID_ARG;
    if (C % 8 != 0) return GTR_ERR_UNSUPPORTED;   // rows of 16-byte multiples (TMA strides)
    if (!aligned16(G) || !aligned16(U) || !aligned16(out) || (reinterpret_cast<uintptr_t>(w) & 3u) ||
        (bias && (reinterpret_cast<uintptr_t>(bias) & 3u)))
        return GTR_ERR_INVALID_ARG;
    if (n > 0x7fffffffLL * 8) return GTR_ERR_INVALID_ARG;
    {   // out may be G itself (each element is read and written by one thread), never U
        const uintptr_t o = reinterpret_cast<uintptr_t>(out), u = reinterpret_cast<uintptr_t>(U);
        const uintptr_t g = reinterpret_cast<uintptr_t>(G), nb = (uintptr_t)n * 2;
        if (o < u + nb && u < o + nb) return GTR_ERR_INVALID_ARG;
        if (o != g && o < g + nb && g < o + nb) return GTR_ERR_INVALID_ARG;
    }
    const int dev = current_device();
    sw::Args a{};
    const gtr_status_t ms = cuda_status(swiglu_maps(G, U, out, B, H, W, C, dev, &a));
    if (ms != GTR_OK) return ms;
    a.w = w;
    a.bias = bias;
    a.B = B;
    a.H = H;
    a.W = W;
    a.C = C;
    a.tiles_x = (W + sw::kTX - 1) / sw::kTX;
    a.tiles_y = (H + sw::kTY - 1) / sw::kTY;
    a.tiles_c = (C + sw::kTC - 1) / sw::kTC;
    const long long tiles = (long long)B * a.tiles_y * a.tiles_x * a.tiles_c;
    if (tiles > 0x7fffffffLL) return GTR_ERR_INVALID_ARG;
    a.tiles = (int)tiles;
    // one tile per CTA with one stage (two CTAs per SM: measured faster), or persistent
    // CTAs with two stages (one per SM) with GTR_SWIGLU=persistent (tuning knob)
    const char *mode = getenv("GTR_SWIGLU");
    const bool persistent = mode && !strcmp(mode, "persistent");
    const int sms = num_sms(dev);
    const long long ctas = persistent ? (tiles < sms ? tiles : sms) : tiles;
    const void *fn = persistent ? reinterpret_cast<const void *>(&sw::swiglu_gate_kernel<2>)
                                : reinterpret_cast<const void *>(&sw::swiglu_gate_kernel<1>);
    const int smem = persistent ? sw::L<2>::alloc : sw::L<1>::alloc;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_status(e);
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1];
    cfg.gridDim = dim3((unsigned)ctas, 1, 1);
    cfg.blockDim = dim3(sw::kThreads, 1, 1);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = reinterpret_cast<cudaStream_t>(stream);
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // set-up overlaps the call ahead
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void *args[] = {&a};
    return cuda_status(cudaLaunchKernelExC(&cfg, fn, args));
}
