/*
 * moe.h -- C ABI of the B200 (sm_100a) routed MoE layer forward.
 *
 * The layer (vLLM fused-MoE page, section 02 "what the fused MoE kernel
 * computes"; the same route -> dispatch -> expert FFN -> combine path as the
 * Weave review, section 1.2, and the stepwise-vs-fused comparison page,
 * section 2):
 *
 *   logit[t,e] = sum_h x[t,h] * router_w[h,e]  (+ router_bias[e])
 *   S_t        = top_k experts by logit, descending; equal logits -> lower index
 *   gate[t,j]  = softmax of the logits of S_t (over the k chosen experts)
 *   out[t]     = sum_j gate[t,j] * W_down[e] ( silu(W_gate[e] x_t) * (W_up[e] x_t) ),
 *                e = S_t[j],  silu(a) = a / (1 + exp(-a))
 *
 * The router logit is an fp32 value with a fixed evaluation order -- a chain of
 * fused multiply-adds over h ascending starting from 0, then + bias[e] in fp32 --
 * so the routing decision is reproducible bit for bit by any implementation
 * that follows the same order.
 *
 * Conventions shared by every call
 *  - Pointers are DEVICE pointers unless stated otherwise; the caller owns all
 *    memory, including the workspace.  The library never allocates or frees
 *    device memory and never synchronises, except moe_get_device_status() and
 *    moe_noalloc_get_device_status().
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    All work is enqueued asynchronously on it; calls on one workspace must not
 *    overlap on the GPU.
 *  - Layouts (row-major, element type in brackets):
 *      x          [T, H]     bf16
 *      router_w   [H, E]     bf16
 *      router_bias[E]        fp32, may be NULL
 *      w_gate     [E, I, H]  bf16 (each expert's rows are K-major, nn.Linear style)
 *      w_up       [E, I, H]  bf16
 *      w_down     [E, H, I]  bf16
 *      out        [T, H]     bf16
 *      topk_idx   [T, top_k] int32,  topk_w [T, top_k] fp32
 *    The flat assignment index of (t, j) is f = t*top_k + j.
 *  - Host-detectable errors return at once and enqueue nothing:
 *      MOE_ERR_INVALID_ARG  NULL dims or required pointer, T < 0, H/I/E <= 0,
 *                           top_k < 1 or > E, H or I not a multiple of 64,
 *                           x, router_w, the expert weights or out not 16-byte aligned
 *      MOE_ERR_UNSUPPORTED  E > 1024
 *      MOE_ERR_WORKSPACE    ws NULL/misaligned (256 B) or ws_bytes too small
 *      MOE_ERR_CUDA         a launch failed (cudaGetLastError)
 *    T == 0 is a no-op that returns MOE_OK.
 *  - Errors found on the device (an expert index outside [0,E) handed to
 *    moe_permute, a pipeline wait that exceeded its time limit) are recorded in
 *    a status word inside the workspace; moe_route, moe_permute and the
 *    forwards clear it when they start, and moe_get_device_status() reads it.
 *  - Results do not depend on the number of GEMM CTAs or on the order in which
 *    they claim work: every sum is taken in an order fixed by the data alone.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,
    MOE_ERR_UNSUPPORTED = 2,
    MOE_ERR_WORKSPACE = 3,
    MOE_ERR_CUDA = 4,
    MOE_ERR_TIMEOUT = 5,     /* device: a pipeline wait ran past its limit */
    MOE_ERR_BAD_INDEX = 6,   /* device: an expert index outside [0, E) */
    MOE_ERR_TOO_LARGE = 7,   /* moe_forward_noalloc: dims need more than its fixed scratch */
    MOE_ERR_ROUTER_BOUND = 8 /* device: a tensor-core router logit fell outside its error bound */
} moe_status_t;

typedef struct {
    int32_t T;      /* tokens */
    int32_t H;      /* hidden size */
    int32_t I;      /* expert intermediate size */
    int32_t E;      /* experts */
    int32_t top_k;  /* experts per token */
} moe_dims_t;

enum { MOE_DTYPE_BF16 = 0, MOE_DTYPE_FP8 = 1, MOE_DTYPE_MX = 2 };

/* Rows of the GEMM tiles; tile_list entries cover at most this many rows. */
#define MOE_TILE_ROWS 128

/* Bytes of workspace every call below needs for these dims (256-byte aligned
 * base required).  Returns 0 for invalid dims.  The workspace holds the router
 * logits, the permutation scratch, the expert-sorted activations and the
 * intermediate h and per-assignment outputs. */
size_t moe_workspace_size(const moe_dims_t *d, int dtype);

/* Upper bound of the number of tile_list entries moe_permute can produce:
 * ceil(T*top_k / 128) + min(E, T*top_k). */
int32_t moe_max_tiles(const moe_dims_t *d);

/* Router logits, top-k selection and softmax gating (vLLM fused-MoE page,
 * section 02: each token's router picks the top-k experts; the k outputs are
 * later summed with these gating weights).
 *   x, router_w, router_bias (nullable)  ->  topk_idx [T,k] int32 (descending
 *   logit, ties to the lower index), topk_w [T,k] fp32 (sums to 1 per token).
 * For T > 32 the logits are first computed on the tensor cores and the fp32
 * chain is evaluated only for the experts within a rounding-error bound of the
 * k-th choice; the result is that of the chain definition.  A chain value found
 * outside its bound records MOE_ERR_ROUTER_BOUND in the status word. */
moe_status_t moe_route(const moe_dims_t *d, const void *x, const void *router_w,
                       const float *router_bias, int32_t *topk_idx, float *topk_w,
                       void *ws, size_t ws_bytes, void *stream);

/* Permute: group the flat assignments by expert (vLLM fused-MoE page, section
 * 02: tokens are sorted and grouped by expert before the grouped GEMM).  A
 * stable counting sort by expert of f = 0..T*k-1:
 *   expert_offsets [E+1]  group e occupies sorted rows [off[e], off[e+1]), no padding
 *   sorted_to_flat [T*k]  flat index of each sorted row (ascending within a group)
 *   flat_to_sorted [T*k]  inverse permutation
 *   tile_list [3*moe_max_tiles]  {expert, row_start, rows} for e ascending and
 *                         each 128-row block of group e (rows <= 128)
 *   num_tiles [1]         number of tile_list entries (device int32)
 * topk_idx entries outside [0,E) are skipped and flagged MOE_ERR_BAD_INDEX. */
moe_status_t moe_permute(const moe_dims_t *d, const int32_t *topk_idx, int32_t *expert_offsets,
                         int32_t *sorted_to_flat, int32_t *flat_to_sorted, int32_t *tile_list,
                         int32_t *num_tiles, void *ws, size_t ws_bytes, void *stream);

/* The whole layer: route, permute, grouped gate/up GEMM with SwiGLU, grouped
 * down GEMM, gate-weighted combine (stepwise-vs-fused comparison page, section
 * 2: two linear layers with SwiGLU per expert between dispatch and combine).
 * Expert GEMMs run on the tensor cores with fp32 accumulation; the SwiGLU
 * output h and the per-assignment expert outputs are rounded to bf16; the
 * combine sums the k contributions in fp32 in ascending j and rounds to bf16. */
moe_status_t moe_forward(const moe_dims_t *d, const void *x, const void *router_w,
                         const float *router_bias, const void *w_gate, const void *w_up,
                         const void *w_down, void *out, void *ws, size_t ws_bytes, void *stream);

/* The layer with a shared expert (GC-MoE page, compute-partition section: the
 * block-scaled expert kernel with "optional shared experts" fused in).  Besides the
 * k routed experts, every token passes through one shared SwiGLU expert with gate
 * weight 1:
 *   out[t] = sum_j gate[t,j] * FFN_{S_t[j]}(x_t)  +  W_sd ( silu(W_sg x_t) * (W_su x_t) )
 *   shared_gate, shared_up [shared_I, H] bf16, shared_down [H, shared_I] bf16.
 * shared_I must be a positive multiple of I (0 = no shared expert: moe_forward).  The
 * shared expert runs inside the same two grouped GEMM launches as the routed ones,
 * as shared_I / I further "experts" of I columns each that every token is routed to;
 * its per-slice outputs are rounded to bf16 like the routed experts' and added after
 * the gate-weighted routed sum (fp32, slices in order), then out is rounded to bf16.
 * The workspace must hold moe_workspace_size_shared(d, shared_I) bytes; other rules
 * as moe_forward.  bf16 only. */
size_t moe_workspace_size_shared(const moe_dims_t *d, int32_t shared_I);
moe_status_t moe_forward_shared(const moe_dims_t *d, const void *x, const void *router_w,
                                const float *router_bias, const void *w_gate, const void *w_up,
                                const void *w_down, int32_t shared_I, const void *shared_gate,
                                const void *shared_up, const void *shared_down, void *out, void *ws,
                                size_t ws_bytes, void *stream);

/* FP8 block-scaled layer (GC-MoE page: block-scaled FP8 MMA on Blackwell with
 * SwiGLU and requantisation fused; vLLM fused-MoE page, section 03: fp8 weights
 * in [128,128] blocks).  Routing is the bf16 router of moe_route.  Weights are
 * e4m3 codes (uint8, OCP "fn" encoding) with one fp32 scale per 128x128 block:
 *   w_gate_q / w_up_q [E, I, H] with w_gate_s / w_up_s [E, I/128, H/128],
 *   w_down_q [E, H, I] with w_down_s [E, H/128, I/128].
 * x (bf16) is quantised per token per 128 columns: s = amax/448 (s = 1 for an
 * all-zero group), q = e4m3 round-to-nearest-even of clamp(v/s, -448, 448);
 * each GEMM is sum over 128-wide K blocks of s_x * s_w * (codes . codes) in fp32
 * on the tensor cores (kind::f8f6f4) with the scaling applied per K block; h =
 * silu(gate) * up is requantised the same way; the down GEMM's per-assignment
 * rows are rounded to bf16 and combined as in moe_forward; out is bf16.
 * Needs H and I multiples of 128 and ws_bytes >= moe_workspace_size(d,
 * MOE_DTYPE_FP8); other rules as moe_forward. */
moe_status_t moe_forward_fp8(const moe_dims_t *d, const void *x, const void *router_w,
                             const float *router_bias, const uint8_t *w_gate_q, const float *w_gate_s,
                             const uint8_t *w_up_q, const float *w_up_s, const uint8_t *w_down_q,
                             const float *w_down_s, void *out, void *ws, size_t ws_bytes, void *stream);

/* MX (microscaling) layer with FP4 weights (GC-MoE page, compute-partition
 * section: block-scaled FP8/FP4 MMAs on Blackwell with the operands swapped and
 * SwiGLU and requantisation fused).  Formats of the OCP Microscaling spec: weights
 * are e2m1 codes, two per byte (the code of element 2i in the low nibble of byte i,
 * of element 2i+1 in the high nibble), with one e8m0 scale code per 32 elements
 * along K; the scale of a block is 2^(code - 127):
 *   w_gate_p / w_up_p [E, I, H/2] with w_gate_x / w_up_x [E, I, H/32],
 *   w_down_p [E, H, I/2] with w_down_x [E, H, I/32]   (uint8).
 * x (bf16) is quantised per token per 32 columns to MX e4m3: X = floor(log2 amax)
 * - 8 clamped to [-127, 127] (X = 0 and zero codes for an all-zero block), codes =
 * e4m3 round-to-nearest-even of clamp(v / 2^X, -448, 448), scale code X + 127.
 * Each GEMM is the sum over 32-wide K blocks of 2^(Xa + Xw) * (codes . codes),
 * accumulated in fp32 on the tensor cores (kind::mxf8f6f4 with block scaling); h
 * = silu(gate) * up (fp32) is requantised to MX e4m3 the same way; the down GEMM's
 * per-assignment rows are rounded to bf16 and combined as in moe_forward.  Routing
 * is the bf16 router of moe_route.  Needs H and I multiples of 512 and ws_bytes >=
 * moe_workspace_size(d, MOE_DTYPE_MX); other rules as moe_forward. */
moe_status_t moe_forward_mx(const moe_dims_t *d, const void *x, const void *router_w,
                            const float *router_bias, const uint8_t *w_gate_p, const uint8_t *w_gate_x,
                            const uint8_t *w_up_p, const uint8_t *w_up_x, const uint8_t *w_down_p,
                            const uint8_t *w_down_x, void *out, void *ws, size_t ws_bytes, void *stream);

/* The activation quantiser of moe_forward_mx on its own: a [R, K] bf16 (K a
 * multiple of 32, 16-byte aligned) -> q [R, K] e4m3 codes and x [R, K/32] e8m0 scale
 * codes, per row per 32 columns as described above.  Needs no workspace. */
moe_status_t moe_quantize_rows_mx(int32_t R, int32_t K, const void *a, uint8_t *q, uint8_t *x, void *stream);

/* The activation quantiser of moe_forward_fp8 on its own: a [R, K] bf16 (K a
 * multiple of 128, 16-byte aligned) -> q [R, K] e4m3 codes and s [R, K/128]
 * fp32 scales, per row per 128 columns as described above.  Needs no workspace. */
moe_status_t moe_quantize_rows_fp8(int32_t R, int32_t K, const void *a, uint8_t *q, float *s, void *stream);

/* Where the last moe_route / moe_forward / moe_forward_fp8 on this workspace
 * left its routing, for inspection: out[i] receives the byte offset of
 *   0 topk_idx [T,k] int32    1 topk_w [T,k] fp32      2 expert_offsets [E+1]
 *   3 sorted_to_flat [T*k]    4 flat_to_sorted [T*k]    5 tile_list [3*max_tiles]
 *   6 num_tiles [1]           7 logits [T,E] fp32
 *   8 xs: the activations in expert-sorted order [T*k, H] (bf16, or 1-byte codes
 *     for MOE_DTYPE_FP8 / MOE_DTYPE_MX; a bf16 forward whose plan has
 *     MOE_PLAN_DIRECT_A does not write it)   9 their scales (fp8: fp32 [T*k, H/128];
 *     MX: e8m0 codes [T*k, H/32])   10 h [T*k, I] (same types)   11 h's scales
 *   12 y [T*k, H] bf16, the per-assignment expert outputs in flat order
 * (0-6 as the outputs of moe_route and moe_permute; 0-1 after moe_route only
 * when it was given the workspace's own regions).  Entry 7 holds the router's
 * fp32 chain value (bias included) of every (t,e) when T <= 32, and of at least
 * each token's chosen experts when T > 32.  Writes min(n, 13) entries; returns
 * MOE_ERR_INVALID_ARG for invalid dims or dtype. */
moe_status_t moe_workspace_offsets(const moe_dims_t *d, int dtype, size_t *out, int32_t n);

/* The kernels a forward with these dims and dtype launches under the current
 * process-wide settings, as bits: the two-kernel router + grouping for small batches,
 * pair-of-CTA GEMM tiles, the combine inside the down GEMM, both expert GEMMs in
 * one launch, and gate/up A rows gathered straight from x (no sorted copy).  -1 for
 * invalid dims or dtype.  Host only; enqueues nothing. */
enum {
    MOE_PLAN_SMALL_ROUTER = 1,
    MOE_PLAN_PAIR_TILES = 2,
    MOE_PLAN_FUSED_COMBINE = 4,
    MOE_PLAN_LAYER_GEMM = 8,
    MOE_PLAN_DIRECT_A = 16
};
int32_t moe_forward_plan(const moe_dims_t *d, int dtype);

/* Synchronises `stream`, returns the device status word of the workspace
 * (MOE_OK, MOE_ERR_TIMEOUT, MOE_ERR_BAD_INDEX or MOE_ERR_ROUTER_BOUND -- the first
 * error recorded since the word was last cleared; MOE_ERR_CUDA if the stream
 * reports an error) and clears it. */
moe_status_t moe_get_device_status(void *ws, void *stream);

/* Number of persistent CTAs each grouped GEMM launches (0 = one per SM, the
 * default).  Results are bitwise independent of it; it exists so that tests can
 * check that.  Process-wide setting. */
void moe_set_gemm_ctas(int32_t ctas);

/* How the GEMM CTAs get their work items (the (m-tile, n-tile) pairs of the
 * expert groups): 0 = the shared atomic queue in ascending order (default);
 * 1 = the queue in descending order; 2 = a static split, CTA c taking items
 * c, c + grid, ...; 3 = a static expert binding, CTA c taking every item of
 * the experts e with e % grid == c (the fixed expert-to-SM assignment that the
 * Weave review, section 2.2, contrasts with dynamic SM scheduling).  Results
 * are bitwise independent of it; modes 2 and 3 exist to measure what the queue
 * buys.  Process-wide. */
void moe_set_claim_order(int32_t mode);

/* Pair-of-CTA GEMMs (tcgen05 cta_group::2: a 256 x 256 tile per 2-CTA cluster,
 * each CTA loading half the operands).  0 = automatic (the bf16 forward uses
 * them when the batch is not a small one and averages at least 768 rows per
 * expert), 1 = whenever the forward can (tests), 2 = never.  Each output is the
 * same K-ordered tensor-core sum either way; the results stay within the layer's
 * tolerance of the oracle.  Process-wide. */
void moe_set_pair_mma(int32_t mode);

/* The fp8 forward's gate/up GEMM with the MMA operands' roles swapped: 128 weight
 * rows on the MMA's M side and the expert group's token rows, rounded up to 16,
 * on its N side, so the tensor work and the per-K-block promotion follow the
 * group's size instead of a 128-row tile.  0 = automatic (used when the batch
 * averages at most 64 rows per expert), 1 = always (tests), 2 = never.  Both
 * forms compute the same blockwise-scaled sums; the output stays within the fp8
 * layer's tolerance either way.  Process-wide. */
void moe_set_fp8_swap_ab(int32_t mode);

/* Where the bf16 forwards sum the k per-assignment rows of a token: 0 = automatic
 * (inside the down GEMM's epilogue for batches of at most 32 tokens, else a separate
 * combine kernel), 1 = always inside the down GEMM, 2 = always the separate kernel.
 * The sum's order is fixed by j either way, so the result is bitwise the same.
 * Process-wide; for tests and benchmarks. */
void moe_set_fused_combine(int32_t mode);

/* The bf16 forwards' two expert GEMMs in one persistent launch (the layer kernel:
 * every gate/up work item is claimed before any down item, and a down item waits --
 * with a bounded wait -- on a per-m-tile count of the epilogue warps that wrote its
 * h rows) or in two launches.  0 = automatic (one launch), 1 = one launch, 2 = two
 * launches.  Results are bitwise the same.  Process-wide; for tests and benchmarks. */
void moe_set_layer_gemm(int32_t mode);

/* Where the bf16 forwards' gate/up GEMM reads its A rows: straight from x, each
 * 128-row tile gathering its tokens' rows four at a time (TMA tile::gather4), or
 * from a copy of x in expert-sorted order made by a gather kernel first (workspace
 * entry 8).  0 = automatic (straight from x), 1 = straight from x, 2 = the sorted
 * copy.  The A values are the same bf16 rows either way, so results are bitwise the
 * same.  Process-wide; for tests and benchmarks. */
void moe_set_direct_a(int32_t mode);

/* Staging of the certified router's exact chains (batches of more than 32 tokens):
 * the block's x rows and router rows pass through shared memory in chunks of
 * 64 * boxes values of h, several chunks in flight.  max_stages caps the chunks in
 * flight (1..8), min_stages is the count the widest chunk must still leave (else the
 * chunk narrows), max_boxes (1, 2, 4 or 8) caps the chunk width; each argument <= 0
 * keeps its default (3, 2, 8).  Every chunk costs the chain phase a barrier of the
 * CTA, so the default takes the widest chunk that leaves two stages.  The chains and so the routing are the same either
 * way.  Process-wide; for tests and benchmarks. */
void moe_set_cert_staging(int32_t max_stages, int32_t min_stages, int32_t max_boxes);

/* Scheduling trace for benchmarks.  With `trace` a device buffer of 4 * ctas
 * uint64 values (ctas >= the GEMM grid, 148 by default), every later forward
 * records per GEMM CTA the %globaltimer (ns) when it started work and when it
 * finished: [2c], [2c + 1] for the gate/up GEMM, [2 ctas + 2c], [2 ctas + 2c + 1]
 * for the down GEMM.  NULL turns it off.  Process-wide. */
void moe_set_gemm_trace(unsigned long long *trace, int32_t ctas);

/* Failure-detection test hook.  Every wait inside the grouped GEMM pipelines
 * is bounded; `us` sets that bound in microseconds (<= 0: the default, 2 s).
 * With `stall_test` nonzero, the MMA thread of every GEMM CTA first waits on a
 * barrier that nothing ever signals, so its wait -- and then the waits of the
 * other roles -- run out.  A wait that runs out makes the kernel record
 * MOE_ERR_TIMEOUT in the workspace status word and unwind (its own TMA copies
 * and MMAs are drained under the default bound before TMEM is freed), so the
 * context stays usable.  Process-wide; for tests only. */
void moe_set_wait_limit_us(int32_t us, int32_t stall_test);

/* Router audit hook for tests.  With `logits` and `bounds` device buffers of at
 * least `capacity` fp32 values, every later certified router run (batches of more
 * than 32 tokens, T*E <= capacity) also writes, for every (t, e), the tensor-core
 * logit plus bias to logits[t*E + e] and the rounding-error bound it uses for that
 * logit to bounds[t*E + e], so a test can check |chain - logit| <= bound for every
 * pair, chosen or not.  NULL (or capacity <= 0) turns it off.  Process-wide. */
void moe_set_router_audit(float *logits, float *bounds, int64_t capacity);

/* Stage timing hook for benchmarks.  With `events` pointing at MOE_STAGE_EVENTS
 * caller-created cudaEvent_t handles (passed as void*), every later moe_forward
 * records them on its stream at the stage boundaries: [0] start, [1] routed,
 * [2] permuted (groups, tile list, sorted activations), [3] gate/up GEMM done,
 * [4] down GEMM done, [5] combined.  A NULL entry is skipped (an event between
 * two kernels costs the step a few microseconds, so whole-step timing passes only
 * [0] and [5]).  The handles must stay valid while set; events == NULL (or
 * n != MOE_STAGE_EVENTS) turns recording off.  Process-wide. */
#define MOE_STAGE_EVENTS 6
void moe_set_stage_events(void *const *events, int32_t n);

/* The layer forward for callers that cannot allocate device memory (the pages
 * have no counterpart; this is a deployment convenience of this library).
 * Same arguments and result as moe_forward minus the workspace: the scratch is
 * a fixed array of MOE_NOALLOC_SCRATCH_BYTES inside the library's device image,
 * present on every GPU that loads the library until the process exits.  It
 * suits callers whose device memory belongs to an allocator they cannot reach,
 * or that must never allocate on their serving path.
 *  - Dims whose moe_workspace_size exceeds the array are rejected with
 *    MOE_ERR_TOO_LARGE (with H=2048, I=512, E=256, top_k=8 that is above
 *    182 tokens); invalid dims give the same errors as moe_forward.
 *  - The first call made with a device current looks up the array's device
 *    address on that device and keeps it for the life of the process; make that
 *    first call before any stream capture, and make no call after a reset of
 *    that device (cudaDeviceReset), which would leave the kept address stale.
 *  - Nothing is allocated, freed or synchronised.  Every call shares the one
 *    array and leaves its contents behind; the parts that must start at zero
 *    are cleared by each call.  Calls whose GPU work overlaps (other streams,
 *    unordered host threads) race on the array: serialise them.
 *  - Device-side status (a pipeline timeout) is kept in the array's status word;
 *    moe_noalloc_get_device_status reads it. */
#define MOE_NOALLOC_SCRATCH_BYTES (16u << 20)
moe_status_t moe_forward_noalloc(const moe_dims_t *d, const void *x, const void *router_w,
                                 const float *router_bias, const void *w_gate, const void *w_up,
                                 const void *w_down, void *out, void *stream);

/* The device status of moe_forward_noalloc on the current device: synchronises
 * `stream`, then reads and clears the status word of the fixed scratch, as
 * moe_get_device_status does for a workspace.  Returns MOE_OK, a device error
 * (MOE_ERR_TIMEOUT, MOE_ERR_BAD_INDEX) of the last call, or MOE_ERR_CUDA. */
moe_status_t moe_noalloc_get_device_status(void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
