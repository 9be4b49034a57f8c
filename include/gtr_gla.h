/*
 * gtr_gla.h -- C ABI of the GTR token-mixer forward pass on B200 (sm_100a).
 *
 * The operation (GTR news article, tokendh.com, section "线性注意力到底在省什么";
 * GTR: Gated Token Recurrence for Efficient Dense Prediction, abstract):
 * a gated linear attention whose learnable forget gate decays the recurrent
 * state on the key side only, the value-side decay being fixed to 1.  For one
 * (batch b, head h) sequence, over scan positions t = 0 .. N-1:
 *
 *     a_t = exp(g_t)                         g_t <= 0, one value per key channel
 *     S_t = diag(a_t) S_{t-1} + k_t^T v_t    S is dk x dv, S_{-1} = init_state or 0
 *     o_t = q_t S_t
 *
 * The patch grid (Hgrid x Wgrid, token n = y*Wgrid + x) is scanned in one of
 * four orders (same article, section "单向扫描的致命缺陷，以及GTR怎么补"):
 *     GTR_L2R  row-major, each row left to right
 *     GTR_R2L  rows top to bottom, each row right to left (the mirrored grid)
 *     GTR_T2B  column-major, each column top to bottom
 *     GTR_B2T  columns left to right, each column bottom to top
 * The state is carried across rows/columns; the direction only changes which
 * token is visited at scan position t.  Tensors stay in grid order in memory.
 *
 * The forward pass is computed chunkwise, 64 scan positions per chunk, in FP16
 * with FP32 accumulation (same article, section "速度到底快在哪，TensorRT部署做了什么":
 * parallel work inside a chunk, only the chunk-boundary state carried in order).
 *
 * Memory layouts (all device pointers, C-contiguous, 16-byte aligned):
 *     q, k, g : IEEE binary16 [B, N, heads, dk]     N = Hgrid * Wgrid
 *     v, out  : IEEE binary16 [B, N, heads, dv]
 *     init_state, final_state : float32 [B, heads, dk, dv]
 * g is the log-decay itself (already divided by the gate temperature); q is
 * used as given (no scaling, no feature map, no normaliser).
 *
 * Ownership: every buffer belongs to the caller; the library never frees or
 * keeps a pointer after a call returns.  All work is enqueued on `stream`
 * (a cudaStream_t, NULL = legacy default stream).  No call synchronises the host
 * except gtr_gla_device_status and the first gtr_gla_fwd_static call on a device.
 *
 * Workspace: for some shapes (dk = 64 with few sequences) one sequence is split
 * into spans that run on different SMs; they exchange one 16.6 KB aggregate per
 * span through a device workspace.  gtr_gla_fwd uses a workspace cached by the
 * library, one per device (about 5 MB), allocated and zero-filled in stream order
 * (cudaMallocAsync / cudaMemsetAsync on the caller's stream, no host wait) by the
 * first call that needs it, or ahead of time by gtr_gla_init.  gtr_gla_fwd calls on
 * one device must not run concurrently on different streams: such callers use
 * gtr_gla_fwd_ws with one workspace each.
 *
 * Numeric range: the tensor-core operands are fp16, so the running state S (as the
 * fp16 operand of the next chunk), the masked scores of a chunk and the outputs must
 * stay below 65504 in magnitude; g must be <= 0 (the log of a forget gate in (0, 1]).
 * A call whose state, scores or outputs leave that range records GTR_ERR_RANGE in the
 * device error word (read by gtr_gla_device_status); its outputs are then unusable.
 * (For inputs like the pages' -- q scaled by dk^-1/2, unit-variance k and v, decaying
 * gates -- these values stay orders of magnitude below the limit.)
 *
 * Errors: argument checks run on the host before anything is enqueued and
 * return GTR_ERR_INVALID_ARG / GTR_ERR_UNSUPPORTED with nothing launched.
 * A failed launch returns GTR_ERR_CUDA.  Device-side waits are bounded; if one
 * runs out the kernel records GTR_ERR_TIMEOUT in a device error word that
 * gtr_gla_device_status reports.
 */
#ifndef GTR_GLA_H
#define GTR_GLA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t gtr_half_t;   /* IEEE 754 binary16 bit pattern */

typedef enum { GTR_L2R = 0, GTR_R2L = 1, GTR_T2B = 2, GTR_B2T = 3 } gtr_dir_t;

typedef enum {
    GTR_OK = 0,
    GTR_ERR_INVALID_ARG = 1,  /* null/negative/misaligned/overflowing/aliased arguments */
    GTR_ERR_UNSUPPORTED = 2,  /* valid but not built: chunk != 64, dk not in {64,128}, dv != 64 */
    GTR_ERR_CUDA = 3,         /* a CUDA runtime call or kernel launch failed */
    GTR_ERR_TIMEOUT = 4,      /* a bounded device-side wait ran out (see gtr_gla_device_status) */
    GTR_ERR_RANGE = 5         /* a value left the fp16 range (see "Numeric range" above) */
} gtr_status_t;

/*
 * Forward pass of one token-mixer layer call.
 *   q, k, v, g      inputs (device), layouts above; may not alias `out`.
 *   B, heads        batch size and number of heads (>= 1).
 *   Hgrid, Wgrid    patch grid; N = Hgrid*Wgrid >= 0 (N == 0 is a no-op that
 *                   still copies init_state to final_state).
 *   dk, dv          key and value head dims, each 64 or 128.  128 runs as two
 *                   64-wide halves (the recurrence is separable by key channel and
 *                   by value column): two launches for dk = 128 (the second adds
 *                   its output to the first's), two writing disjoint columns for
 *                   dv = 128, four for both.
 *   direction       gtr_dir_t scan order.
 *   chunk           chunk length; 64 (the only value built).
 *   init_state      float32 [B, heads, dk, dv] or NULL for a zero state.
 *   out             float16 [B, N, heads, dv], fully written.
 *   final_state     float32 [B, heads, dk, dv] or NULL; the state after the last
 *                   scan position.  May equal init_state (in-place carry).
 *   stream          cudaStream_t to enqueue on.
 */
gtr_status_t gtr_gla_fwd(const gtr_half_t *q, const gtr_half_t *k, const gtr_half_t *v,
                         const gtr_half_t *g, int B, int heads, int Hgrid, int Wgrid,
                         int dk, int dv, int direction, int chunk,
                         const float *init_state, gtr_half_t *out, float *final_state,
                         void *stream);

/*
 * gtr_gla_fwd with the forget gate given by its pre-activation: the third input z
 * (IEEE binary16 [B, N, heads, dk], in place of g) and the temperature tau > 0; the
 * kernel forms g = log(sigmoid(z)) / tau = (min(z, 0) - log(1 + exp(-|z|))) / tau in
 * fp32 wherever it reads the gate of a chunk (GTR news article, section "线性注意力到底在省什么":
 * a learnable forget gate on the key side), so no separate pass over z runs and g is
 * never rounded to fp16.  Same arguments, layouts, workspace and errors as gtr_gla_fwd,
 * plus GTR_ERR_INVALID_ARG for tau <= 0 or not finite.
 */
gtr_status_t gtr_gla_fwd_z(const gtr_half_t *q, const gtr_half_t *k, const gtr_half_t *v,
                           const gtr_half_t *z, float tau, int B, int heads, int Hgrid, int Wgrid,
                           int dk, int dv, int direction, int chunk,
                           const float *init_state, gtr_half_t *out, float *final_state,
                           void *stream);

/* One layer call of a stack (gtr_gla_fwd_stack): the tensors of gtr_gla_fwd. */
typedef struct {
    const gtr_half_t *q, *k, *v, *g;   /* inputs, layouts as above */
    const float *init_state;           /* float32 [B, heads, dk, dv] or NULL */
    gtr_half_t *out;                   /* float16 [B, N, heads, dv] */
    float *final_state;                /* float32 [B, heads, dk, dv] or NULL */
    int direction;                     /* gtr_dir_t */
} gtr_gla_layer_t;

/*
 * A stack of n_layers token-mixer calls of one shape, in order, on `stream`: the GTR
 * backbone's blocks each scan in one direction, cycling L->R, R->L, T->B, B->T over its
 * twelve blocks (GTR news article, section "单向扫描的致命缺陷，以及GTR怎么补").  Each layer
 * has its own tensors and direction; a layer may read an earlier layer's outputs or
 * final state (stream order).  Consecutive launches overlap (each layer's set-up runs
 * while the previous one drains).  Outside a stream capture the launches are recorded
 * once into a CUDA graph per distinct layer list (pointers, directions, shape), on a
 * private stream of the library's (so `stream` may be the legacy default stream), and
 * that graph is launched on `stream`, so a repeated stack costs one graph launch of
 * host time (the eight most recent layer lists are kept); inside a
 * capture they are simply enqueued into the caller's graph.  Same per-layer arguments,
 * checks and results as gtr_gla_fwd (a failing layer's index is not reported: every
 * layer is checked before anything is enqueued).  1 <= n_layers <= 64.
 * (The pages' model interleaves other operators between these calls; the stack is the
 * token-mixer part of it.)
 */
gtr_status_t gtr_gla_fwd_stack(const gtr_gla_layer_t *layers, int n_layers, int B, int heads,
                               int Hgrid, int Wgrid, int dk, int dv, int chunk, void *stream);

/*
 * Allocates and zero-fills, in the order of `stream` (no host wait), the library's
 * cached workspace of the current device, sized for every shape, so that no later
 * gtr_gla_fwd call allocates.  Call it before capturing gtr_gla_fwd calls into a
 * CUDA graph: a first allocation during a capture returns GTR_ERR_CUDA
 * (cudaErrorStreamCaptureUnsupported) with nothing enqueued.  Calling it again is a
 * no-op.  (No counterpart on the pages: this is the library's memory contract.)
 */
gtr_status_t gtr_gla_init(void *stream);

/*
 * Bytes of workspace gtr_gla_fwd_ws needs for a shape on the current device
 * (0: none needed, or arguments gtr_gla_fwd would reject).  Host-only query.
 */
size_t gtr_gla_workspace_bytes(int B, int heads, int Hgrid, int Wgrid, int dk, int dv, int chunk);

/*
 * gtr_gla_fwd with a caller-owned workspace: same arguments and results, plus
 *   workspace        device memory, 256-byte aligned, at least
 *                    gtr_gla_workspace_bytes(...) bytes (may be NULL when that is 0).
 *                    It must be zero-filled before its first use.  Its first
 *                    part (the spans' publish flags, 2 x 128 bytes per SM of
 *                    the device, rounded up to 256) must be zero when a call starts:
 *                    every call that completes without a device error leaves it
 *                    zero again; the rest holds the spans' aggregates, which any
 *                    call overwrites before reading.  After GTR_ERR_TIMEOUT the
 *                    caller zero-fills the workspace again.
 *   workspace_bytes  its size.
 * Calls that share a workspace must not overlap in time (same stream is fine).
 * A missing, short or misaligned workspace returns GTR_ERR_INVALID_ARG.
 * (No counterpart on the pages: this is the library's memory contract.)
 */
gtr_status_t gtr_gla_fwd_ws(const gtr_half_t *q, const gtr_half_t *k, const gtr_half_t *v,
                            const gtr_half_t *g, int B, int heads, int Hgrid, int Wgrid,
                            int dk, int dv, int direction, int chunk,
                            const float *init_state, gtr_half_t *out, float *final_state,
                            void *workspace, size_t workspace_bytes, void *stream);

/* Size of the library's static device scratch used by gtr_gla_fwd_static: 4 MiB. */
#define GTR_STATIC_WS_BYTES (4u << 20)

/*
 * gtr_gla_fwd that allocates nothing.  The paper has no counterpart: this is a
 * memory-management variant of the library's own call.  Same arguments, results
 * and argument errors as gtr_gla_fwd.  Where the shape's plan needs a workspace
 * (gtr_gla_workspace_bytes > 0), the span kernel's workspace lives in one
 * file-scope device array of GTR_STATIC_WS_BYTES bytes inside the library instead
 * of memory from an allocator; no call makes cudaMalloc, cudaFree or any other
 * allocating call.
 *   - Set-up: the first call on a device that needs the scratch looks up its
 *     device address (cudaGetSymbolAddress) with that device current and
 *     zero-fills its publish flags (the part that must be zero when a call
 *     starts; every call that completes without a device error leaves them
 *     zero again), synchronising the host once.
 *     Make that first call before any stream capture begins.
 *   - Limit: the call picks the cheapest launch plan whose workspace fits in
 *     GTR_STATIC_WS_BYTES (one span per sequence needs none, so every shape that
 *     gtr_gla_fwd accepts runs); only a plan forced past that size by the
 *     GTR_CLUSTER_SIZE tuning variable falls back to another plan.
 *   - The scratch is shared by every gtr_gla_fwd_static call on the device:
 *     calls that overlap in time (different streams or host threads) race on it
 *     and give wrong results.  Calls in order on one stream are fine.
 */
gtr_status_t gtr_gla_fwd_static(const gtr_half_t *q, const gtr_half_t *k, const gtr_half_t *v,
                                const gtr_half_t *g, int B, int heads, int Hgrid, int Wgrid,
                                int dk, int dv, int direction, int chunk,
                                const float *init_state, gtr_half_t *out, float *final_state,
                                void *stream);

/*
 * Syncs `stream`, then reads and clears the device error word (and any sticky
 * CUDA error).  Returns GTR_OK, GTR_ERR_TIMEOUT, GTR_ERR_RANGE or GTR_ERR_CUDA.  On
 * GTR_ERR_TIMEOUT it also zero-fills the library's workspaces of the current
 * device (the cached one and the static scratch).
 */
gtr_status_t gtr_gla_device_status(void *stream);

/*
 * Self-test of the device-side failure path (no counterpart on the pages: this
 * checks the library's own error reporting).  Enqueues on `stream` a one-CTA
 * kernel whose waits (an mbarrier nothing arrives on, a flag nothing sets) run
 * through the same bounded-wait code as the forward kernels, with a limit of
 * limit_us microseconds (1 .. 1000000) instead of their 200 ms.  Both waits run
 * out; the kernel sets the device error word and ends normally, so the next
 * gtr_gla_device_status returns GTR_ERR_TIMEOUT (and clears it), and the context
 * stays usable.  Returns GTR_ERR_INVALID_ARG for a limit out of range, else the
 * launch status.
 */
gtr_status_t gtr_gla_selftest_timeout(unsigned limit_us, void *stream);

/* Static text for a status code (never NULL). */
const char *gtr_status_str(gtr_status_t status);

/*
 * Launch plan the library would use for a shape on the current device:
 * writes the number of CTAs cooperating on one sequence (the spans it is cut
 * into, in `cluster_size`), the number of such CTA groups in the grid and the
 * dynamic shared memory per CTA (a dk = 128 call runs this plan twice, once per
 * 64-channel key half).  Host-only query; returns GTR_ERR_* like gtr_gla_fwd's
 * argument checks.
 */
gtr_status_t gtr_gla_plan(int B, int heads, int Hgrid, int Wgrid, int dk, int dv,
                          int *cluster_size, int *num_clusters, int *smem_bytes);

/*
 * Text of the last CUDA error a gtr_gla_fwd call on this host thread returned
 * GTR_ERR_CUDA for ("no error" if none); static storage, never NULL.
 */
const char *gtr_gla_last_error(void);

/* Library version, "major.minor.patch". */
const char *gtr_gla_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GTR_GLA_H */
