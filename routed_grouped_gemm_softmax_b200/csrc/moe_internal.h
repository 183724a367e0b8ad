// moe_internal.h -- workspace layout and kernel launchers shared by the library's
// translation units (not part of the public ABI).
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/moe.h"

namespace moe {

constexpr int kTileRows = MOE_TILE_ROWS;  // BM of the grouped GEMMs
constexpr int kMaxExperts = 1024;
constexpr int kRouterKSplitMax = 8;  // K slices of the router's tensor-core logits

// Header at the start of every workspace.
struct WsHeader {
    int32_t status;       // device status word (moe_status_t), sticky until read
    int32_t counter[7];   // work-claim counters of the persistent GEMMs
    int32_t pad[8];
};

// Byte offsets of every region of the workspace (256-byte aligned each).
struct WsLayout {
    size_t ccnt, ready, clear_bytes, logits, wrt, wsq, rncand, rlist, blk_cnt, blk_base, idx, gate, offsets, s2f, f2s, tiles, ntiles, tiles2, ntiles2, xq, xq_s, xs, xs_s, h, h_s, y,
        total;
    int nb;      // permutation chunks
    int chunk;   // flat entries per chunk
};

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Entries of the flat assignment list handled by one permutation chunk: the
// scatter kernel keeps a [warps x E] table of per-warp counts in shared memory,
// so wide expert counts use fewer warps.
inline int perm_warps(int E)
{
    int w = 8192 / (E > 0 ? E : 1);
    if (w > 32) w = 32;
    if (w < 1) w = 1;
    return w;
}

// Workspace regions; with fp8 the sorted activations and h are e4m3 codes plus
// one fp32 scale per 128 columns, and x is quantised per token before the gather.
inline WsLayout ws_layout(const moe_dims_t &d, int dtype = MOE_DTYPE_BF16, int sh_count = 0)
{
    const bool fp8 = dtype == MOE_DTYPE_FP8, mx = dtype == MOE_DTYPE_MX;
    // bytes of the scales of n activation values: fp32 per 128 (fp8), e8m0 per 32 (MX)
    auto act_scales = [&](size_t n) { return fp8 ? n / 128 * 4 : mx ? n / 32 : 0; };
    const bool q8 = fp8 || mx;  // one-byte activation codes
    const size_t SR = static_cast<size_t>(sh_count) * d.T;  // shared expert rows of h and y
    WsLayout L{};
    const size_t A = static_cast<size_t>(d.T) * d.top_k;
    const int warps = perm_warps(d.E);
    L.chunk = 32 * warps;
    L.nb = static_cast<int>((A + L.chunk - 1) / L.chunk);
    const size_t max_tiles = (A + kTileRows - 1) / kTileRows + (A < (size_t)d.E ? A : (size_t)d.E);
    size_t o = align_up(sizeof(WsHeader), 256);
    // the fused combine's arrival counts and the fused layer GEMM's per-m-tile
    // readiness counts follow the header, so one memset clears all three
    const size_t mtiles = (A + kTileRows - 1) / kTileRows + (A < (size_t)d.E ? A : (size_t)d.E) +
                          static_cast<size_t>(sh_count) * ((d.T + kTileRows - 1) / kTileRows);
    L.ccnt = o;
    L.ready = L.ccnt + static_cast<size_t>(d.T) * ((d.H + 255) / 256) * 4;
    L.clear_bytes = L.ready + mtiles * 4;
    o = align_up(L.clear_bytes, 1024);
    auto take = [&](size_t bytes) {
        size_t at = o;
        o = align_up(o + bytes, 1024);
        return at;
    };
    L.logits = take(static_cast<size_t>(d.T) * d.E * 4 * kRouterKSplitMax);
    L.wrt = take(static_cast<size_t>(d.E) * d.H * 2);
    L.wsq = take(static_cast<size_t>(d.E) * 4 * ((d.H + 255) / 256));  // partial squared norms
    const bool tc_router = d.T > 32;  // the certified router's candidate lists
    L.rncand = take(tc_router ? static_cast<size_t>(d.T) * 4 : 0);
    L.rlist = take(tc_router ? static_cast<size_t>(d.T) * d.E * 16 : 0);
    L.blk_cnt = take(static_cast<size_t>(L.nb > 0 ? L.nb : 1) * d.E * 4);
    L.blk_base = take(static_cast<size_t>(L.nb > 0 ? L.nb : 1) * d.E * 4);
    L.idx = take(A * 4);
    L.gate = take(A * 4);
    L.offsets = take(static_cast<size_t>(d.E + 1) * 4);
    L.s2f = take(A * 4);
    L.f2s = take(A * 4);
    L.tiles = take(max_tiles * 3 * 4);
    L.ntiles = take(4);
    L.tiles2 = take(((A + 2 * kTileRows - 1) / (2 * kTileRows) + (A < (size_t)d.E ? A : (size_t)d.E)) * 3 * 4);
    L.ntiles2 = take(4);
    L.xq = take(q8 ? static_cast<size_t>(d.T) * d.H : 0);  // fp8 / MX: x quantised once per token
    L.xq_s = take(act_scales(static_cast<size_t>(d.T) * d.H));
    L.xs = take(A * d.H * (q8 ? 1 : 2));
    L.xs_s = take(act_scales(A * d.H));
    L.h = take((A + SR) * d.I * (q8 ? 1 : 2));
    L.h_s = take(act_scales(A * d.I));
    L.y = take((A + SR) * d.H * 2);
    L.total = o;
    return L;
}

// ------------------------------------------------------------ launchers
// Each returns cudaGetLastError() of its launch(es).

// Candidate of the certified router: token, expert, tensor-core logit (+bias), bound.
struct RouterCand {
    int t, e;
    float v, d;
};

// Scratch of the certified router (T > 32).
struct RouterScratch {
    __nv_bfloat16 *wrt;  // [E, H] router matrix, transposed
    float *wsq;          // [ceil(H/256), E] partial squared column norms
    int32_t *ncand;      // [T] candidates per token
    RouterCand *list;    // [T, E] candidates of each token, ascending expert index
    float *audit_v;      // test hook, or null: [T, E] tensor-core logit (+bias) of every (t, e)
    float *audit_d;      // test hook, or null: [T, E] its rounding-error bound
};

// Router: for T <= 32 the CUDA-core fp32 chains (route.cu); above, tensor-core
// logits certified against the chains (route_certified.cu).  Uses work counter 2
// and the status word.
cudaError_t launch_route(const moe_dims_t &d, const __nv_bfloat16 *x, const __nv_bfloat16 *wr,
                         const float *bias, float *logits, int32_t *idx, float *gate,
                         const RouterScratch &rs, WsHeader *hdr, cudaStream_t st);
cudaError_t launch_route_certified(const moe_dims_t &d, const __nv_bfloat16 *x, const __nv_bfloat16 *wr,
                                   const float *bias, float *logits, int32_t *idx, float *gate,
                                   const RouterScratch &rs, WsHeader *hdr, cudaStream_t st);

// Router + permute in two launches for small batches (T <= 32, E % 8 == 0,
// H % 128 == 0, T*k <= 4096, ceil(T*k/32) * E <= 16384).  They also clear the
// workspace header (status word, work counters) and the nccnt combine counts,
// so a forward on this path needs no memset.
bool small_route_permute_ok(const moe_dims_t &d);
cudaError_t launch_route_permute_small(const moe_dims_t &d, const __nv_bfloat16 *x, const __nv_bfloat16 *wr,
                                       const float *bias, float *logits, int32_t *idx, float *gate,
                                       int32_t *offsets, int32_t *s2f, int32_t *f2s, int32_t *tiles,
                                       int32_t *ntiles, WsHeader *hdr, int32_t *ccnt, int nccnt, cudaStream_t st);

// Also writes the 2 x 128-row pair tiles when tiles2 is non-null.
cudaError_t launch_permute(const moe_dims_t &d, const WsLayout &L, const int32_t *idx,
                           int32_t *blk_cnt, int32_t *blk_base, int32_t *offsets, int32_t *s2f,
                           int32_t *f2s, int32_t *tiles, int32_t *ntiles, WsHeader *hdr,
                           cudaStream_t st, int32_t *tiles2 = nullptr, int32_t *ntiles2 = nullptr);

// xs[f2s[f]] = x[f / k] for every assignment f = t*k + j (a warp per assignment, flat order).
cudaError_t launch_gather_rows(const __nv_bfloat16 *x, const int32_t *f2s, int T, int H, int top_k,
                               __nv_bfloat16 *xs, cudaStream_t st);


// Grouped GEMMs over the tile list.  mode 0: h = silu(A Wg^T) * (A Wu^T) (A = the
// expert-sorted activations, B = gate/up weights); mode 1: y[s2f[row]] = A Wd^T
// (A = h).  The tensor maps are encoded by the caller.
// Tensor maps of one A operand with boxes of 16, 32, 64 and 128 rows: a tile loads
// only the smallest box that covers its rows (the rest of its shared-memory tile is
// left as it is; those output rows are masked).
constexpr int kABoxes = 4;
struct AMaps {
    CUtensorMap m[kABoxes];
};
__host__ __device__ inline int a_box(int rows) { return rows <= 16 ? 0 : rows <= 32 ? 1 : rows <= 64 ? 2 : 3; }
__host__ __device__ inline int a_box_rows(int b) { return 16 << b; }

struct GemmArgs {
    int mode;
    int K, N;
    const int32_t *tiles;
    const int32_t *ntiles;
    int32_t *counter;
    int32_t *status;
    __nv_bfloat16 *out;
    const int32_t *row_map;
    int ctas;
    int reverse;       // claim mode: 0/1 queue ascending/descending, 2 static items, 3 static experts
    uint64_t wait_ns;  // limit of each pipeline wait
    int stall_test;    // MMA thread first waits on a barrier nothing signals
    int M;             // mode 2 (no tile list): rows of A
    float *out_f32;    // mode 2: fp32 output [M, N]
    // mode 1, fused combine (comb_cnt non-null): after its y rows of an n-tile are
    // written, the last of the comb_target arrivals for (token, n-tile) sums the
    // token's k rows of that n-tile into comb_out.
    const float *comb_gate;
    int32_t *comb_cnt;            // [T, ceil(N / 256)], zero before the launch
    __nv_bfloat16 *comb_out;      // [T, N]
    int comb_k;
    int comb_target;
    unsigned long long *trace;  // per CTA {start, end} globaltimer (ns), or null
    // Shared expert (modes 0 and 1; sh_count = 0: none).  Its intermediate width is
    // sh_count * I, cut into sh_count slices of I: slice s is one more "expert",
    // number sh_e0 + s, that every token passes through with gate 1.  Its m-tiles
    // follow the tile list's: block i of slice s covers the h / y rows
    // sh_rows0 + s * sh_T + [i * BM, min((i + 1) * BM, sh_T)), whose A rows are the
    // token rows i * BM.. of x in mode 0 (SharedMaps::x) and those h rows in mode 1;
    // its weights come from SharedMaps::b0 / b1 (2-D maps over the whole shared
    // matrices, slice s at row s * I (gate/up) or column s * I (down)).  In mode 1
    // these y rows are written in place (no row map), after the T * k routed rows.
    int sh_count;
    int sh_T;
    int sh_rows0;
    int sh_e0;
    // Mode 3, the gate/up and the down GEMM in one persistent launch: the gate/up items
    // (K, N, out = h) come first in the claim order, then the down items (K2, N2, out2
    // = y, row_map, fused combine as in mode 1).  A down item of m-tile mt waits (at
    // most wait_ns) until ready[mt] counts the 4 epilogue warps of every gate/up item
    // of mt (2 x 4 for pair tiles), then reads those h rows.  ready is zeroed before
    // the launch.
    int K2, N2;
    __nv_bfloat16 *out2;
    int32_t *ready;
    // Gate/up items of routed tiles with a_rows non-null: the A rows are read straight
    // from x (SharedMaps::xg, one-row boxes) by tile::gather4 loads, row r of a tile
    // being token a_rows[row0 + r] / a_div (no expert-ordered copy of x is made); a
    // token outside [0, a_tokens) reads row 0 instead.
    const int32_t *a_rows;
    int a_div, a_tokens;
    // The tile list is written by the kernel launched just before this one (no other
    // kernel in between), so it is read only after the programmatic-dependency wait.
    int tiles_first;
};

// Tensor maps of the down half of the fused layer GEMM (mode 3): h as its A operand
// (16 to 128-row boxes), the down weights (3-D) and the shared expert's (2-D).
struct LayerMaps {
    AMaps h;
    CUtensorMap wd, wd_sh;
};

// Tensor maps of the shared expert: x as the gate/up GEMM's A operand (boxes of 16
// to 128 rows), and the gate/up (b0, b1: [sh_count * I, H]) or down (b0: [H,
// sh_count * I]) weights as 2-D maps.  Unused (zero) without a shared expert.
struct SharedMaps {
    AMaps x;
    CUtensorMap b0, b1;
    CUtensorMap xg;  // x with one-row boxes of 64 columns (128-byte swizzle), for tile::gather4 A loads
};

// The m-tile `mt` of a grouped GEMM: the tile list's entry for mt < nrouted, else a
// block of the shared expert (GemmArgs::sh_*), for tiles of `bm` rows.
struct TileRef {
    int e, row0, rows;  // expert, first h/y row, rows
    int arow0;          // first A row (x row of a shared tile in mode 0, else row0)
    int s;              // shared slice, or -1
};
__device__ __forceinline__ TileRef tile_ref(const int32_t *tiles, int nrouted, int mt, int bm, int mode, int sh_T,
                                            int sh_rows0, int sh_e0)
{
    TileRef r;
    if (mt < nrouted) {
        r.e = tiles[3 * mt];
        r.row0 = tiles[3 * mt + 1];
        r.rows = tiles[3 * mt + 2];
        r.arow0 = r.row0;
        r.s = -1;
        return r;
    }
    const int tps = (sh_T + bm - 1) / bm, q = mt - nrouted;
    const int i = q % tps;
    r.s = q / tps;
    r.e = sh_e0 + r.s;
    r.row0 = sh_rows0 + r.s * sh_T + i * bm;
    r.rows = min(bm, sh_T - i * bm);
    r.arow0 = mode == 0 ? i * bm : r.row0;
    return r;
}
// mode 2: out_f32 = A B^T over M rows (one "expert"), the router's tensor-core logits.
cudaError_t launch_grouped_gemm(const GemmArgs &g, const AMaps &tmA, const CUtensorMap &tmB0,
                                const CUtensorMap &tmB1, cudaStream_t st, const SharedMaps *sm = nullptr,
                                const LayerMaps *lm = nullptr);

// The bf16 grouped GEMMs (modes 0 and 1) on CTA pairs, cta_group::2 MMAs over the
// 2 x 128-row pair tiles tiles2 (grouped_gemm_2cta.cu); queue claim modes only.
cudaError_t launch_grouped_gemm_2cta(const GemmArgs &g, const AMaps &tmA, const CUtensorMap &tmB0,
                                     const CUtensorMap &tmB1, const int32_t *tiles2, const int32_t *ntiles2,
                                     cudaStream_t st, const SharedMaps *sm = nullptr, const LayerMaps *lm = nullptr);

// FP8 block-scaled grouped GEMMs (fp8.cu).  mode 0: h codes/scales from
// silu(A Wg^T) * (A Wu^T); mode 1: y[row_map[row]] = A Wd^T in bf16; mode 2:
// bf16 A B^T summed per 64-wide K block into fp32 partials (router logits).
struct Fp8GemmArgs {
    int mode;
    int K, N;
    const int32_t *tiles;
    const int32_t *ntiles;
    int32_t *counter;
    int32_t *status;
    const float *sa;   // activation scales [rows, K/128]
    const float *sb0;  // weight scales [E, N/128, K/128] (gate or down)
    const float *sb1;  // up scales (mode 0)
    uint8_t *out_q;    // mode 0: h codes [rows, N]
    float *out_s;      // mode 0: h scales [rows, N/128]
    __nv_bfloat16 *out;      // mode 1: y [T*k, N]
    const int32_t *row_map;  // mode 1: sorted row -> flat row
    int ctas;
    int reverse;  // claim mode, as in GemmArgs
    uint64_t wait_ns;
    int stall_test;
    int M;            // mode 2: rows of A (no tile list)
    int ksplit;       // mode 2: items per (m-tile, n-tile), each a slice of K
    float *out_f32;   // mode 2: partial logits [ksplit, M, N]
    const float *comb_gate;  // mode 1 fused combine, as in GemmArgs
    int32_t *comb_cnt;
    __nv_bfloat16 *comb_out;
    int comb_k;
    int comb_target;
    unsigned long long *trace;  // per CTA {start, end} globaltimer (ns), or null
};
cudaError_t launch_grouped_gemm_fp8(const Fp8GemmArgs &g, const AMaps &tmA, const CUtensorMap &tmB0,
                                    const CUtensorMap &tmB1, cudaStream_t st);
// The fp8 gate/up GEMM (mode 0 only) with the MMA operands swapped: 128 weight rows
// on the M side, the tile's token rows (rounded up to 16) on the N side
// (fp8_swapab.cu); for expert groups much shorter than a 128-row tile.
cudaError_t launch_grouped_gemm_fp8_swapab(const Fp8GemmArgs &g, const AMaps &tmX, const CUtensorMap &tmWg,
                                           const CUtensorMap &tmWu, cudaStream_t st);
cudaError_t launch_quantize_rows(const __nv_bfloat16 *src, const int32_t *map, int k, int R, int K, uint8_t *q,
                                 float *s, cudaStream_t st);
// fp8 rows into expert order: xs[r] = xq[s2f[r] / k] (K codes) and xs_s[r] = xq_s[...] (K/128 scales).
cudaError_t launch_gather_rows_fp8(const uint8_t *xq, const float *xq_s, const int32_t *s2f, int A, int K, int k,
                                   uint8_t *xs, float *xs_s, cudaStream_t st);

// MX grouped GEMMs (mx.cu): e2m1 weights x e4m3 activations with e8m0 scales per 32
// along K, block-scaled on the tensor cores, operands swapped (weight rows on M).
// mode 0: h codes/scale codes from silu(X Wg^T) * (X Wu^T); mode 1: y[row_map[row]]
// = X Wd^T in bf16.  K a multiple of 512, N of 128.  Tensor maps: tmX the token
// rows' codes (16/32/64-row boxes), tmW0/tmW1 the two 128-row weight tiles of an item
// (16U4_ALIGN16B, 3-D), tmSX the token rows' scale codes (64 x 16 boxes), tmSW0/tmSW1
// the weight scale codes (3-D, 128 x 16 boxes).
struct MxLaunch {
    int mode, K, N;
    const int32_t *tiles, *ntiles;
    int32_t *counter, *status;
    uint8_t *out_q, *out_x;
    __nv_bfloat16 *out;
    const int32_t *row_map;
    int ctas, reverse;
    uint64_t wait_ns;
    int stall_test;
    unsigned long long *trace;
    AMaps tmX;
    CUtensorMap tmW0, tmW1, tmSX, tmSW0, tmSW1;
};
cudaError_t launch_grouped_gemm_mx(const MxLaunch &l, cudaStream_t st);
// MX e4m3 codes and e8m0 scale codes (per 32 columns) of bf16 rows [R, K].
cudaError_t launch_quantize_rows_mx(const __nv_bfloat16 *src, int R, int K, uint8_t *q, uint8_t *x, cudaStream_t st);
// MX rows into expert order: xs[r] = xq[s2f[r] / k], xs_x[r] = xq_x[s2f[r] / k].
cudaError_t launch_gather_rows_mx(const uint8_t *xq, const uint8_t *xq_x, const int32_t *s2f, int A, int K, int k,
                                  uint8_t *xs, uint8_t *xs_x, cudaStream_t st);

// Tensor-core router logits: partial sums over ksplit slices of H,
// logits [ksplit, T, E] with sum_s logits[s] = x [T,H] . wrt [E,H]^T (fp32 per
// 64-wide K block, then fp32 sums).  Returns ksplit through *ksplit_out.
cudaError_t tc_router_logits(const __nv_bfloat16 *x, const __nv_bfloat16 *wrt, int T, int H, int E, float *logits,
                             WsHeader *hdr, int *ksplit_out, cudaStream_t st);

// Gate-weighted combine of the k per-assignment rows of every token (combine.cu),
// plus, with sh_count > 0, the shared expert's rows y[sh_rows0 + s * T + t] at gate 1.
cudaError_t launch_combine(const __nv_bfloat16 *y, const float *gate, int T, int H, int top_k,
                           __nv_bfloat16 *out, cudaStream_t st, int sh_count = 0, int sh_rows0 = 0);
// ----------------------------------------------------------- tile table
// The kernel variants by M bucket: the batch's average rows per expert r = T*k/E (the
// vLLM fused-MoE page keys its tuned configs by M the same way, section 03).  Measured
// on B200 with CUDA events (H=2048, I=1024, E=64, top-8, r = 1 .. 4096, uniform
// routing; and the Skewed workload, r = 768 with a Zipf-skewed router, at 1x and 2x
// its tokens):
//  - pair-of-CTA 256-row tiles lose 3-8% to 128-row tiles below r = 512 and win from
//    r = 2048 (uniform); on the skewed workload they win at r = 768 (1.68 against
//    1.72 ms) and r = 1536 (5.6%), its deep hot-expert groups filling the pairs;
//  - one persistent launch for both GEMMs (the layer kernel) wins 6-14% below r = 512
//    and on the skewed workload, and is within 1-3% elsewhere;
//  - the fp8 gate/up GEMM with the operands swapped wins up to r = 64 (up to 40%) and
//    loses from r = 96 (up to 2x at r = 1024).
// Each entry covers the buckets up to max_rows.
struct TileChoice {
    int max_rows;     // the bucket: average rows per expert <= max_rows
    bool pair_tiles;  // bf16: 256-row tiles on CTA pairs (tcgen05 cta_group::2)
    bool layer_gemm;  // bf16: the gate/up and down GEMMs in one launch
    bool fp8_swap_ab; // fp8: gate/up GEMM with the weight rows on the MMA's M side
    bool direct_a;    // bf16: gate/up A rows gathered straight from x (no sorted copy)
};
constexpr TileChoice kTileTable[] = {
    {16, false, true, true, true},
    {64, false, true, true, false},
    {767, false, true, false, false},
    {0x7fffffff, true, true, false, false},
};
inline TileChoice tile_choice(long long A, int E)
{
    const long long r = E > 0 ? A / E : A;  // average rows per expert, rounded down
    for (const TileChoice &t : kTileTable)
        if (r <= t.max_rows) return t;
    return kTileTable[sizeof(kTileTable) / sizeof(kTileTable[0]) - 1];
}
// Batches up to this many tokens combine inside the down GEMM's epilogue (the sweep:
// 1% faster at T <= 16, even at 32, 4% slower at 64 and 20-30% slower from 256).
constexpr int kFusedCombineMaxT = 32;
// The fp8 down GEMM's fused combine (two epilogue warps per row) keeps its own limit.
constexpr int kFusedCombineMaxTFp8 = 64;

int num_sms();

// Tensor map of a row-major bf16 matrix [rows, cols], box_rows x 64 tiles with the
// 128-byte swizzle (16-byte chunk c of tile row r stored at chunk c ^ (r % 8)).
bool encode_sw128_2d_bf16(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows);
// The same matrix seen as [cols / 64][rows][64]: one box brings box_chunks consecutive
// 64-column chunks of box_rows rows, stored chunk after chunk (each chunk's rows as the
// 2-D map's box would store them).
bool encode_sw128_chunked_bf16(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows,
                               uint32_t box_chunks);
// Tensor map of a row-major bf16 matrix [rows, cols], box_rows x box_cols tiles,
// no swizzle (box_cols * 2 a multiple of 16).
bool encode_plain_2d_bf16(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                          uint32_t box_rows);

}  // namespace moe
