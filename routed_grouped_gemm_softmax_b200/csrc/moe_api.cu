// moe_api.cu -- the C ABI declared in include/moe.h: argument checks, workspace
// carving, TMA descriptor encoding and the launch sequence of the layer.
//
// moe_forward enqueues, on the caller's stream:
//   route_logits -> route_topk          (router, softmax over the top-k)
//   perm_count -> perm_scan -> perm_scatter   (group assignments by expert)
//   gather_rows                         (activations in expert-sorted order)
//   grouped GEMM mode 0                 (gate/up + SwiGLU -> h)
//   grouped GEMM mode 1                 (down -> one row per assignment)
//   combine                             (gate-weighted sum back to token order)
// following the route -> dispatch -> expert FFN -> combine stages of the
// stepwise-vs-fused comparison page (section 6, stepwise pseudo-code), on one GPU.
#include <atomic>
#include <cstring>
#include <mutex>

#include "moe_internal.h"

namespace {

std::atomic<int> g_gemm_ctas{0};
std::atomic<int> g_claim_reverse{0};
std::atomic<unsigned long long *> g_trace{nullptr};
std::atomic<int> g_pair_mode{0};  // 0 auto, 1 pair GEMMs whenever possible, 2 never
std::atomic<int> g_fp8_swap{0};   // 0 auto, 1 swapped fp8 gate/up GEMM always, 2 never
std::atomic<int> g_fused_comb{0}; // 0 auto, 1 combine inside the down GEMM always, 2 never
std::atomic<int> g_layer_gemm{0}; // 0 auto, 1 gate/up and down GEMMs in one launch always, 2 never
std::atomic<int> g_cert_max_stages{0}, g_cert_min_stages{0}, g_cert_max_boxes{0};  // 0: defaults
std::atomic<int> g_direct_a{0};   // 0 auto, 1 gate/up A rows gathered straight from x always, 2 never
std::atomic<int> g_trace_ctas{0};
std::atomic<unsigned long long> g_wait_ns{0};
std::atomic<int> g_stall_test{0};
std::mutex g_audit_mu;
float *g_audit_v = nullptr, *g_audit_d = nullptr;  // router audit buffers (test hook)
int64_t g_audit_cap = 0;
std::mutex g_ev_mu;
cudaEvent_t g_stage_ev[MOE_STAGE_EVENTS];
bool g_stage_on = false;

struct StageMarks {
    cudaEvent_t ev[MOE_STAGE_EVENTS];
    bool on = false;
    StageMarks()
    {
        std::lock_guard<std::mutex> lk(g_ev_mu);
        on = g_stage_on;
        for (int i = 0; i < MOE_STAGE_EVENTS; ++i) ev[i] = g_stage_ev[i];
    }
    // While the stream is being captured into a CUDA graph, external records become
    // event-record nodes, so a replayed graph still timestamps every stage; otherwise
    // the events are recorded directly (the external flag is for captures only).
    cudaError_t mark(int i, cudaStream_t st) const
    {
        if (!on || !ev[i]) return cudaSuccess;
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return cudaErrorInvalidValue;
        return cs == cudaStreamCaptureStatusActive ? cudaEventRecordWithFlags(ev[i], st, cudaEventRecordExternal)
                                                   : cudaEventRecord(ev[i], st);
    }
};

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// bf16 matrix [rows, cols] (row-major), tiles of box_rows x 64 with the 128-byte swizzle.
bool encode_2d(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows)
{
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t es[2] = {1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 weights [E, rows, cols], tiles of box_rows x 64 of one expert.
// e4m3 matrix [rows, cols] bytes, tiles of box_rows x 128 bytes with the 128-byte swizzle.
bool encode_2d_u8(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows)
{
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols};
    const cuuint32_t box[2] = {128, box_rows};
    const cuuint32_t es[2] = {1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// e4m3 weights [E, rows, cols] bytes, tiles of box_rows x 128 bytes of one expert.
bool encode_3d_u8(CUtensorMap *m, const void *base, uint64_t E, uint64_t rows, uint64_t cols, uint32_t box_rows)
{
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    const cuuint64_t dims[3] = {cols, rows, E};
    const cuuint64_t strides[2] = {cols, rows * cols};
    const cuuint32_t box[3] = {128, box_rows, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 partial logits [ks][M][N] as 32-column x 32-row boxes with the 128-byte swizzle,
// for tensor-map stores (N a multiple of 4, so that rows are 16-byte aligned).
bool encode_logits_store(CUtensorMap *m, float *base, uint64_t ks, uint64_t M, uint64_t N)
{
    EncodeTiledFn f = encode_fn();
    if (!f || N % 4) return false;
    const cuuint64_t dims[3] = {N, M, ks};
    const cuuint64_t strides[2] = {N * 4, M * N * 4};
    const cuuint32_t box[3] = {32, 32, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// e2m1 weights [E, rows, cols], packed two codes per byte, seen as [E][cols / 128][rows]
// [128 codes]: one box brings two consecutive 128-code chunks of box_rows rows (128
// contiguous packed bytes a row, where a single chunk reads 64), chunk after chunk. TMA
// expands every 16 codes to 16 bytes (the MMA's 4-bit operand layout) under the 128-byte
// swizzle.
bool encode_4d_fp4_pairs(CUtensorMap *m, const void *base, uint64_t E, uint64_t rows, uint64_t cols,
                         uint32_t box_rows)
{
    EncodeTiledFn f = encode_fn();
    if (!f || cols % 256) return false;
    const cuuint64_t dims[4] = {128, rows, cols / 128, E};
    const cuuint64_t strides[3] = {cols / 2, 64, rows * cols / 2};
    const cuuint32_t box[4] = {128, box_rows, 2, 1};
    const cuuint32_t es[4] = {1, 1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 4, const_cast<void *>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Scale codes (bytes) [E, rows, cols], boxes of 16 codes x box_rows, no swizzle: a
// 3-D map (rank 3, loaded with 3 coordinates) or, with rank 2, a 2-D one over [rows,
// cols] (E = 1).
bool encode_scales_u8(CUtensorMap *m, const void *base, uint64_t E, uint64_t rows, uint64_t cols, uint32_t box_rows,
                      int rank)
{
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    const cuuint64_t dims[3] = {cols, rows, E};
    const cuuint64_t strides[2] = {cols, rows * cols};
    const cuuint32_t box[3] = {16, box_rows, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    if (rank != 3 && !(rank == 2 && E == 1)) return false;
    return f(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, (cuuint32_t)rank, const_cast<void *>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_3d(CUtensorMap *m, const void *base, uint64_t E, uint64_t rows, uint64_t cols, uint32_t box_rows)
{
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    const cuuint64_t dims[3] = {cols, rows, E};
    const cuuint64_t strides[2] = {cols * 2, rows * cols * 2};
    const cuuint32_t box[3] = {64, box_rows, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 weights [E, rows, cols] seen as [E][cols / 64][rows][64]: one box brings kc
// consecutive 64-column chunks of box_rows rows of one expert, chunk after chunk, so
// each row is read 128 * kc contiguous bytes at a time (DRAM streams such boxes about
// a third faster than 128-byte row pieces).
bool encode_4d_chunked(CUtensorMap *m, const void *base, uint64_t E, uint64_t rows, uint64_t cols, uint32_t box_rows,
                       uint32_t kc)
{
    EncodeTiledFn f = encode_fn();
    if (!f || cols % 64) return false;
    const cuuint64_t dims[4] = {64, rows, cols / 64, E};
    const cuuint64_t strides[3] = {cols * 2, 128, rows * cols * 2};
    const cuuint32_t box[4] = {64, box_rows, kc, 1};
    const cuuint32_t es[4] = {1, 1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

moe_status_t check_dims(const moe_dims_t *d)
{
    if (!d) return MOE_ERR_INVALID_ARG;
    if (d->T < 0 || d->H <= 0 || d->I <= 0 || d->E <= 0) return MOE_ERR_INVALID_ARG;
    if (d->top_k < 1 || d->top_k > d->E) return MOE_ERR_INVALID_ARG;
    if (d->H % 64 != 0 || d->I % 64 != 0) return MOE_ERR_INVALID_ARG;
    if (d->E > moe::kMaxExperts) return MOE_ERR_UNSUPPORTED;
    if ((int64_t)d->T * d->top_k > (int64_t)INT32_MAX / 2) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

moe_status_t check_ws(const moe_dims_t *d, const void *ws, size_t ws_bytes)
{
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_WORKSPACE;
    if (ws_bytes < moe::ws_layout(*d).total) return MOE_ERR_WORKSPACE;
    return MOE_OK;
}

template <class T>
T *at(void *ws, size_t off)
{
    return reinterpret_cast<T *>(static_cast<uint8_t *>(ws) + off);
}

moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

moe::RouterScratch router_scratch(void *ws, const moe::WsLayout &L, const moe_dims_t &d)
{
    moe::RouterScratch rs{at<__nv_bfloat16>(ws, L.wrt), at<float>(ws, L.wsq), at<int32_t>(ws, L.rncand),
                          at<moe::RouterCand>(ws, L.rlist), nullptr, nullptr};
    std::lock_guard<std::mutex> lk(g_audit_mu);
    if (g_audit_v && (int64_t)d.T * d.E <= g_audit_cap) {
        rs.audit_v = g_audit_v;
        rs.audit_d = g_audit_d;
    }
    return rs;
}

// The bf16 forward's choice of kernels for these dims under the current settings
// (MOE_PLAN_* bits).
int bf16_plan(const moe_dims_t &d)
{
    const moe::TileChoice tc = moe::tile_choice((long long)d.T * d.top_k, d.E);
    const bool small = moe::small_route_permute_ok(d);
    const int pair_mode = g_pair_mode.load();
    const bool pairs = pair_mode != 2 && g_claim_reverse.load() <= 1 && !small && (pair_mode == 1 || tc.pair_tiles);
    const int fc = g_fused_comb.load();
    const bool fused = fc == 1 || (fc == 0 && d.T <= moe::kFusedCombineMaxT);
    const int lg = g_layer_gemm.load();
    const bool layer = lg == 1 || (lg == 0 && tc.layer_gemm);
    const int da = g_direct_a.load();
    const bool direct = da == 1 || (da == 0 && tc.direct_a);
    return (small ? MOE_PLAN_SMALL_ROUTER : 0) | (pairs ? MOE_PLAN_PAIR_TILES : 0) |
           (fused ? MOE_PLAN_FUSED_COMBINE : 0) | (layer ? MOE_PLAN_LAYER_GEMM : 0) | (direct ? MOE_PLAN_DIRECT_A : 0);
}

// Activations, weights and outputs are read and written in 16-byte vectors (and the
// weights by TMA, which needs 16-byte aligned bases).
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Router and permute: one fused launch for small batches, otherwise the logits,
// top-k and three permute kernels.  Stage mark 1 (routed) is recorded between the
// two in the multi-kernel form and together with the fused launch otherwise.
cudaError_t route_and_permute(const moe_dims_t &d, const moe::WsLayout &L, const void *x, const void *router_w,
                              const float *router_bias, void *ws, moe::WsHeader *hdr, const StageMarks &marks,
                              cudaStream_t st)
{
    auto *idx = at<int32_t>(ws, L.idx);
    auto *gate = at<float>(ws, L.gate);
    auto *s2f = at<int32_t>(ws, L.s2f);
    auto *tiles = at<int32_t>(ws, L.tiles);
    auto *ntiles = at<int32_t>(ws, L.ntiles);
    const auto *xb = static_cast<const __nv_bfloat16 *>(x);
    const auto *wb = static_cast<const __nv_bfloat16 *>(router_w);
    if (moe::small_route_permute_ok(d)) {
        cudaError_t e = moe::launch_route_permute_small(d, xb, wb, router_bias, at<float>(ws, L.logits), idx, gate,
                                                        at<int32_t>(ws, L.offsets), s2f, at<int32_t>(ws, L.f2s),
                                                        tiles, ntiles, hdr, at<int32_t>(ws, L.ccnt),
                                                        (int)((L.clear_bytes - L.ccnt) / 4), st);
        return e == cudaSuccess ? marks.mark(1, st) : e;
    }
    cudaError_t e =
        moe::launch_route(d, xb, wb, router_bias, at<float>(ws, L.logits), idx, gate, router_scratch(ws, L, d), hdr, st);
    if (e == cudaSuccess) e = marks.mark(1, st);
    if (e == cudaSuccess)
        e = moe::launch_permute(d, L, idx, at<int32_t>(ws, L.blk_cnt), at<int32_t>(ws, L.blk_base),
                                at<int32_t>(ws, L.offsets), s2f, at<int32_t>(ws, L.f2s), tiles, ntiles, hdr, st,
                                at<int32_t>(ws, L.tiles2), at<int32_t>(ws, L.ntiles2));
    return e;
}

}  // namespace

namespace moe {
// bf16 matrix [rows, cols] (row-major), tiles of box_rows x box_cols, no swizzle.
bool encode_plain_2d_bf16(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                          uint32_t box_rows)
{
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t es[2] = {1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 matrix [rows, cols], tiles of box_rows x 64 with the 128-byte swizzle.
bool encode_sw128_2d_bf16(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows)
{
    return encode_2d(m, base, rows, cols, box_rows);
}

bool encode_sw128_chunked_bf16(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows,
                               uint32_t box_chunks)
{
    EncodeTiledFn f = encode_fn();
    if (!f || cols % 64) return false;
    const cuuint64_t dims[3] = {64, rows, cols / 64};
    const cuuint64_t strides[2] = {cols * 2, 128};  // a row, a 64-column chunk
    const cuuint32_t box[3] = {64, box_rows, box_chunks};
    const cuuint32_t es[3] = {1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A-operand tensor maps with boxes of 16/32/64/128 rows (bf16 64 columns, or 128
// e4m3 bytes), 128-byte swizzle.
bool encode_a_maps(AMaps *m, const void *base, uint64_t rows, uint64_t cols, bool u8)
{
    for (int b = 0; b < kABoxes; ++b) {
        const uint32_t br = (uint32_t)a_box_rows(b);
        if (!(u8 ? encode_2d_u8(&m->m[b], base, rows, cols, br) : encode_2d(&m->m[b], base, rows, cols, br)))
            return false;
    }
    return true;
}

void cert_staging(int *max_stages, int *min_stages, int *max_boxes)
{
    *max_stages = g_cert_max_stages.load();
    *min_stages = g_cert_min_stages.load();
    *max_boxes = g_cert_max_boxes.load();
}

// The router's tensor-core logits: the block-promoting GEMM (fp8.cu, mode 2, bf16
// operands) over plain 128-row blocks of x against the transposed router matrix,
// K split over enough items to occupy the GPU, the partial logits stored by tensor
// map from the stage buffers once a CTA's items are done.  The items are uniform, so
// they are dealt out statically (no work counter, and so nothing between the router's prep
// kernel and this one: x loads overlap the prep kernel's tail).
cudaError_t tc_router_logits(const __nv_bfloat16 *x, const __nv_bfloat16 *wrt, int T, int H, int E, float *logits,
                             WsHeader *hdr, int *ksplit_out, cudaStream_t st)
{
    AMaps tm_x;
    CUtensorMap tm_w;
    if (!encode_a_maps(&tm_x, x, T, H, false) || !encode_3d(&tm_w, wrt, 1, E, H, 256)) return cudaErrorInvalidValue;
    const int items = ((T + kTileRows - 1) / kTileRows) * ((E + 255) / 256);
    int ks = (120 + items - 1) / items;
    ks = ks < 1 ? 1 : ks > kRouterKSplitMax ? kRouterKSplitMax : ks;
    if (ks > H / 64) ks = H / 64;
    *ksplit_out = ks;
    Fp8GemmArgs g{2, H, E, nullptr, nullptr, &hdr->counter[2], &hdr->status, nullptr, nullptr, nullptr, nullptr,
                  nullptr, nullptr, nullptr, 0, 2, 2000000000ull, 0, T, ks, logits};
    // with E a multiple of 4 the epilogue stores the partial logits through this map
    // (passed as the kernel's third map, which mode 2 does not otherwise use)
    CUtensorMap tm_out = tm_w;
    if (E % 4 == 0 && !encode_logits_store(&tm_out, logits, (uint64_t)ks, (uint64_t)T, (uint64_t)E))
        return cudaErrorInvalidValue;
    return launch_grouped_gemm_fp8(g, tm_x, tm_w, tm_out, st);
}
}  // namespace moe

extern "C" {

size_t moe_workspace_size(const moe_dims_t *d, int dtype)
{
    if (check_dims(d) != MOE_OK) return 0;
    if (dtype == MOE_DTYPE_FP8) {
        if (d->H % 128 || d->I % 128) return 0;
        return moe::ws_layout(*d, MOE_DTYPE_FP8).total;
    }
    if (dtype == MOE_DTYPE_MX) {
        if (d->H % 512 || d->I % 512) return 0;
        return moe::ws_layout(*d, MOE_DTYPE_MX).total;
    }
    if (dtype != MOE_DTYPE_BF16) return 0;
    return moe::ws_layout(*d).total;
}

int32_t moe_max_tiles(const moe_dims_t *d)
{
    if (check_dims(d) != MOE_OK) return 0;
    const int64_t A = (int64_t)d->T * d->top_k;
    return (int32_t)((A + moe::kTileRows - 1) / moe::kTileRows + (A < d->E ? A : d->E));
}

void moe_set_gemm_ctas(int32_t ctas) { g_gemm_ctas.store(ctas > 0 ? ctas : 0); }

void moe_set_claim_order(int32_t mode) { g_claim_reverse.store(mode < 0 ? 0 : mode > 3 ? 3 : mode); }

void moe_set_pair_mma(int32_t mode) { g_pair_mode.store(mode < 0 || mode > 2 ? 0 : mode); }
void moe_set_fp8_swap_ab(int32_t mode) { g_fp8_swap.store(mode < 0 || mode > 2 ? 0 : mode); }
void moe_set_fused_combine(int32_t mode) { g_fused_comb.store(mode < 0 || mode > 2 ? 0 : mode); }
void moe_set_layer_gemm(int32_t mode) { g_layer_gemm.store(mode < 0 || mode > 2 ? 0 : mode); }

void moe_set_direct_a(int32_t mode) { g_direct_a.store(mode < 0 || mode > 2 ? 0 : mode); }

void moe_set_cert_staging(int32_t max_stages, int32_t min_stages, int32_t max_boxes)
{
    g_cert_max_stages.store(max_stages > 0 ? (max_stages > 8 ? 8 : max_stages) : 0);
    g_cert_min_stages.store(min_stages > 0 ? (min_stages > 8 ? 8 : min_stages) : 0);
    g_cert_max_boxes.store(max_boxes >= 8 ? 8 : max_boxes >= 4 ? 4 : max_boxes >= 2 ? 2 : max_boxes == 1 ? 1 : 0);
}

void moe_set_gemm_trace(unsigned long long *trace, int32_t ctas)
{
    g_trace.store(trace && ctas > 0 ? trace : nullptr);
    g_trace_ctas.store(ctas > 0 ? ctas : 0);
}

void moe_set_wait_limit_us(int32_t us, int32_t stall_test)
{
    g_wait_ns.store(us > 0 ? static_cast<unsigned long long>(us) * 1000ull : 0ull);
    g_stall_test.store(stall_test ? 1 : 0);
}

void moe_set_router_audit(float *logits, float *bounds, int64_t capacity)
{
    std::lock_guard<std::mutex> lk(g_audit_mu);
    const bool on = logits && bounds && capacity > 0;
    g_audit_v = on ? logits : nullptr;
    g_audit_d = on ? bounds : nullptr;
    g_audit_cap = on ? capacity : 0;
}

void moe_set_stage_events(void *const *events, int32_t n)
{
    std::lock_guard<std::mutex> lk(g_ev_mu);
    g_stage_on = events != nullptr && n == MOE_STAGE_EVENTS;
    for (int i = 0; i < MOE_STAGE_EVENTS; ++i)
        g_stage_ev[i] = g_stage_on ? static_cast<cudaEvent_t>(events[i]) : nullptr;
}

moe_status_t moe_route(const moe_dims_t *d, const void *x, const void *router_w, const float *router_bias,
                       int32_t *topk_idx, float *topk_w, void *ws, size_t ws_bytes, void *stream)
{
    moe_status_t s = check_dims(d);
    if (s != MOE_OK) return s;
    if (d->T == 0) return MOE_OK;
    if (!x || !router_w || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(router_w)) return MOE_ERR_INVALID_ARG;
    if ((s = check_ws(d, ws, ws_bytes)) != MOE_OK) return s;
    const moe::WsLayout L = moe::ws_layout(*d);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(int32_t), st);
    if (e == cudaSuccess)
        e = moe::launch_route(*d, static_cast<const __nv_bfloat16 *>(x), static_cast<const __nv_bfloat16 *>(router_w),
                              router_bias, at<float>(ws, L.logits), topk_idx, topk_w, router_scratch(ws, L, *d),
                              at<moe::WsHeader>(ws, 0), st);
    return cuda_status(e);
}

moe_status_t moe_permute(const moe_dims_t *d, const int32_t *topk_idx, int32_t *expert_offsets,
                         int32_t *sorted_to_flat, int32_t *flat_to_sorted, int32_t *tile_list,
                         int32_t *num_tiles, void *ws, size_t ws_bytes, void *stream)
{
    moe_status_t s = check_dims(d);
    if (s != MOE_OK) return s;
    if (d->T == 0) return MOE_OK;
    if (!topk_idx || !expert_offsets || !sorted_to_flat || !flat_to_sorted || !tile_list || !num_tiles)
        return MOE_ERR_INVALID_ARG;
    if ((s = check_ws(d, ws, ws_bytes)) != MOE_OK) return s;
    const moe::WsLayout L = moe::ws_layout(*d);
    cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(int32_t), static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    return cuda_status(moe::launch_permute(*d, L, topk_idx, at<int32_t>(ws, L.blk_cnt),
                                           at<int32_t>(ws, L.blk_base), expert_offsets, sorted_to_flat,
                                           flat_to_sorted, tile_list, num_tiles, at<moe::WsHeader>(ws, 0),
                                           static_cast<cudaStream_t>(stream)));
}

size_t moe_workspace_size_shared(const moe_dims_t *d, int32_t shared_I)
{
    if (check_dims(d) != MOE_OK || shared_I < 0 || shared_I % d->I != 0) return 0;
    return moe::ws_layout(*d, MOE_DTYPE_BF16, shared_I / d->I).total;
}

moe_status_t moe_forward(const moe_dims_t *d, const void *x, const void *router_w, const float *router_bias,
                         const void *w_gate, const void *w_up, const void *w_down, void *out, void *ws,
                         size_t ws_bytes, void *stream)
{
    return moe_forward_shared(d, x, router_w, router_bias, w_gate, w_up, w_down, 0, nullptr, nullptr, nullptr, out,
                              ws, ws_bytes, stream);
}

moe_status_t moe_forward_shared(const moe_dims_t *d, const void *x, const void *router_w, const float *router_bias,
                                const void *w_gate, const void *w_up, const void *w_down, int32_t shared_I,
                                const void *shared_gate, const void *shared_up, const void *shared_down, void *out,
                                void *ws, size_t ws_bytes, void *stream)
{
    moe_status_t s = check_dims(d);
    if (s != MOE_OK) return s;
    if (shared_I < 0 || shared_I % d->I != 0) return MOE_ERR_INVALID_ARG;
    const int sh = shared_I / d->I;  // slices of the shared expert, I columns each
    if (d->T == 0) return MOE_OK;
    if (!x || !router_w || !w_gate || !w_up || !w_down || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(router_w) || !aligned16(w_gate) || !aligned16(w_up) || !aligned16(w_down) ||
        !aligned16(out))
        return MOE_ERR_INVALID_ARG;
    if (sh && (!shared_gate || !shared_up || !shared_down || !aligned16(shared_gate) || !aligned16(shared_up) ||
               !aligned16(shared_down)))
        return MOE_ERR_INVALID_ARG;
    if ((int64_t)sh * d->T + (int64_t)d->T * d->top_k > (int64_t)INT32_MAX / 2) return MOE_ERR_UNSUPPORTED;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_WORKSPACE;
    const moe::WsLayout L = moe::ws_layout(*d, MOE_DTYPE_BF16, sh);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int A = d->T * d->top_k;
    const int R = A + sh * d->T;  // rows of h and y: the routed assignments, then the shared expert's
    auto *hdr = at<moe::WsHeader>(ws, 0);
    auto *xs = at<__nv_bfloat16>(ws, L.xs);
    auto *h = at<__nv_bfloat16>(ws, L.h);
    auto *y = at<__nv_bfloat16>(ws, L.y);
    auto *gate = at<float>(ws, L.gate);
    auto *s2f = at<int32_t>(ws, L.s2f);
    auto *tiles = at<int32_t>(ws, L.tiles);
    auto *ntiles = at<int32_t>(ws, L.ntiles);

    moe::AMaps tm_xs, tm_h;
    CUtensorMap tm_wg, tm_wu, tm_wd;
    // pair-of-CTA GEMMs for groups large enough to be compute-bound (on average at
    // least 768 rows per expert), on the queue's claim modes
    const int plan = bf16_plan(*d);
    const bool pairs = plan & MOE_PLAN_PAIR_TILES;
    if (!moe::encode_a_maps(&tm_xs, xs, A, d->H, false) ||
        !encode_4d_chunked(&tm_wg, w_gate, d->E, d->I, d->H, 128, 2) ||
        !encode_4d_chunked(&tm_wu, w_up, d->E, d->I, d->H, 128, 2) ||
        !moe::encode_a_maps(&tm_h, h, R, d->I, false) ||
        !encode_4d_chunked(&tm_wd, w_down, d->E, d->H, d->I, pairs ? 128 : 256, 2))
        return MOE_ERR_CUDA;
    // the shared expert: x itself as its gate/up A operand, its weights as chunked maps
    // with the boxes of the routed experts' maps
    moe::SharedMaps sm1{}, sm2{};
    if (sh && (!moe::encode_a_maps(&sm1.x, x, d->T, d->H, false) ||
               !moe::encode_sw128_chunked_bf16(&sm1.b0, shared_gate, shared_I, d->H, 128, 2) ||
               !moe::encode_sw128_chunked_bf16(&sm1.b1, shared_up, shared_I, d->H, 128, 2) ||
               !moe::encode_sw128_chunked_bf16(&sm2.b0, shared_down, d->H, shared_I, pairs ? 128 : 256, 2)))
        return MOE_ERR_CUDA;
    // gate/up A rows straight from x: one-row boxes for tile::gather4, the token of
    // sorted row r being sorted_to_flat[r] / k
    const bool direct = plan & MOE_PLAN_DIRECT_A;
    if (direct && !encode_2d(&sm1.xg, x, d->T, d->H, 1)) return MOE_ERR_CUDA;
    // the tile list is then the output of the kernel just before the gate/up GEMM
    // when the router and the grouping are one launch
    const int tiles_first = direct && (plan & MOE_PLAN_SMALL_ROUTER) ? 1 : 0;

    const StageMarks marks;
    const bool fused = plan & MOE_PLAN_FUSED_COMBINE;  // combine inside the down GEMM
    cudaError_t e = marks.mark(0, st);
    if (e == cudaSuccess && !moe::small_route_permute_ok(*d))  // else the router's kernels clear them
        e = cudaMemsetAsync(hdr, 0, L.clear_bytes, st);          // header + combine counts
    if (e == cudaSuccess) e = route_and_permute(*d, L, x, router_w, router_bias, ws, hdr, marks, st);
    if (e == cudaSuccess && !direct)
        e = moe::launch_gather_rows(static_cast<const __nv_bfloat16 *>(x), at<int32_t>(ws, L.f2s), d->T, d->H,
                                    d->top_k, xs, st);
    if (e == cudaSuccess) e = marks.mark(2, st);
    const int ctas = g_gemm_ctas.load(), rev = g_claim_reverse.load();
    unsigned long long *trace1 = g_trace.load(), *trace2 = trace1 ? trace1 + 2 * g_trace_ctas.load() : nullptr;
    const unsigned long long wl = g_wait_ns.load();
    const uint64_t wait_ns = wl ? wl : 2000000000ull;
    const int stall = g_stall_test.load();
    // the gate/up and the down GEMM in one persistent launch (readiness counters per
    // m-tile hand h from one to the other)
    const bool layer = plan & MOE_PLAN_LAYER_GEMM;
    if (e == cudaSuccess && layer) {
        moe::GemmArgs gl{3, d->H, d->I, tiles, ntiles, &hdr->counter[0], &hdr->status, h, s2f, ctas, rev, wait_ns,
                         stall, 0, nullptr, gate, fused ? at<int32_t>(ws, L.ccnt) : nullptr,
                         static_cast<__nv_bfloat16 *>(out), d->top_k, d->top_k + sh};
        gl.trace = trace1;
        gl.sh_count = sh;
        gl.sh_T = d->T;
        gl.sh_rows0 = A;
        gl.sh_e0 = d->E;
        gl.K2 = d->I;
        gl.N2 = d->H;
        gl.out2 = y;
        gl.ready = at<int32_t>(ws, L.ready);
        if (direct) {
            gl.a_rows = s2f;
            gl.a_div = d->top_k;
            gl.a_tokens = d->T;
            gl.tiles_first = tiles_first;
        }
        moe::LayerMaps lm{};
        lm.h = tm_h;
        lm.wd = tm_wd;
        lm.wd_sh = sm2.b0;
        e = pairs ? moe::launch_grouped_gemm_2cta(gl, tm_xs, tm_wg, tm_wu, at<int32_t>(ws, L.tiles2),
                                                  at<int32_t>(ws, L.ntiles2), st, &sm1, &lm)
                  : moe::launch_grouped_gemm(gl, tm_xs, tm_wg, tm_wu, st, &sm1, &lm);
        if (e == cudaSuccess) e = marks.mark(3, st);
        if (e == cudaSuccess) e = marks.mark(4, st);
    }
    if (e == cudaSuccess && !layer) {
        moe::GemmArgs g1{0, d->H, d->I, tiles, ntiles, &hdr->counter[0], &hdr->status, h, nullptr, ctas, rev, wait_ns, stall};
        g1.trace = trace1;
        g1.sh_count = sh;
        g1.sh_T = d->T;
        g1.sh_rows0 = A;
        g1.sh_e0 = d->E;
        if (direct) {
            g1.a_rows = s2f;
            g1.a_div = d->top_k;
            g1.a_tokens = d->T;
            g1.tiles_first = tiles_first;
        }
        e = pairs ? moe::launch_grouped_gemm_2cta(g1, tm_xs, tm_wg, tm_wu, at<int32_t>(ws, L.tiles2),
                                                  at<int32_t>(ws, L.ntiles2), st, &sm1)
                  : moe::launch_grouped_gemm(g1, tm_xs, tm_wg, tm_wu, st, &sm1);
        if (e == cudaSuccess) e = marks.mark(3, st);
    }
    if (e == cudaSuccess && !layer) {
        moe::GemmArgs g2{1, d->I, d->H, tiles, ntiles, &hdr->counter[1], &hdr->status, y, s2f, ctas, rev, wait_ns,
                         stall, 0, nullptr, gate, fused ? at<int32_t>(ws, L.ccnt) : nullptr,
                         static_cast<__nv_bfloat16 *>(out), d->top_k, d->top_k + sh};
        g2.trace = trace2;
        g2.sh_count = sh;
        g2.sh_T = d->T;
        g2.sh_rows0 = A;
        g2.sh_e0 = d->E;
        e = pairs ? moe::launch_grouped_gemm_2cta(g2, tm_h, tm_wd, tm_wd, at<int32_t>(ws, L.tiles2),
                                                  at<int32_t>(ws, L.ntiles2), st, &sm2)
                  : moe::launch_grouped_gemm(g2, tm_h, tm_wd, tm_wd, st, &sm2);
        if (e == cudaSuccess) e = marks.mark(4, st);
    }
    if (e == cudaSuccess && !fused)
        e = moe::launch_combine(y, gate, d->T, d->H, d->top_k, static_cast<__nv_bfloat16 *>(out), st, sh, A);
    if (e == cudaSuccess) e = marks.mark(5, st);
    return cuda_status(e);
}

moe_status_t moe_quantize_rows_fp8(int32_t R, int32_t K, const void *a, uint8_t *q, float *s, void *stream)
{
    if (R < 0 || K <= 0 || K % 128) return MOE_ERR_INVALID_ARG;
    if (R == 0) return MOE_OK;
    if (!a || !q || !s || !aligned16(a) || !aligned16(q)) return MOE_ERR_INVALID_ARG;
    return cuda_status(moe::launch_quantize_rows(static_cast<const __nv_bfloat16 *>(a), nullptr, 1, R, K, q, s,
                                                 static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_forward_fp8(const moe_dims_t *d, const void *x, const void *router_w, const float *router_bias,
                             const uint8_t *w_gate_q, const float *w_gate_s, const uint8_t *w_up_q,
                             const float *w_up_s, const uint8_t *w_down_q, const float *w_down_s, void *out,
                             void *ws, size_t ws_bytes, void *stream)
{
    moe_status_t s = check_dims(d);
    if (s != MOE_OK) return s;
    if (d->H % 128 || d->I % 128) return MOE_ERR_INVALID_ARG;
    if (d->T == 0) return MOE_OK;
    if (!x || !router_w || !w_gate_q || !w_gate_s || !w_up_q || !w_up_s || !w_down_q || !w_down_s || !out)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(router_w) || !aligned16(w_gate_q) || !aligned16(w_up_q) ||
        !aligned16(w_down_q) || !aligned16(out))
        return MOE_ERR_INVALID_ARG;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_WORKSPACE;
    const moe::WsLayout L = moe::ws_layout(*d, MOE_DTYPE_FP8);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int A = d->T * d->top_k;
    auto *hdr = at<moe::WsHeader>(ws, 0);
    auto *xs = at<uint8_t>(ws, L.xs);
    auto *xs_s = at<float>(ws, L.xs_s);
    auto *h = at<uint8_t>(ws, L.h);
    auto *h_s = at<float>(ws, L.h_s);
    auto *y = at<__nv_bfloat16>(ws, L.y);
    auto *idx = at<int32_t>(ws, L.idx);
    auto *gate = at<float>(ws, L.gate);
    auto *s2f = at<int32_t>(ws, L.s2f);
    auto *tiles = at<int32_t>(ws, L.tiles);
    auto *ntiles = at<int32_t>(ws, L.ntiles);

    moe::AMaps tm_xs, tm_h;
    CUtensorMap tm_wg, tm_wu, tm_wd;
    if (!moe::encode_a_maps(&tm_xs, xs, A, d->H, true) || !encode_3d_u8(&tm_wg, w_gate_q, d->E, d->I, d->H, 128) ||
        !encode_3d_u8(&tm_wu, w_up_q, d->E, d->I, d->H, 128) || !moe::encode_a_maps(&tm_h, h, A, d->I, true) ||
        !encode_3d_u8(&tm_wd, w_down_q, d->E, d->H, d->I, 256))
        return MOE_ERR_CUDA;

    const StageMarks marks;
    const bool fused = d->T <= moe::kFusedCombineMaxTFp8;  // combine inside the down GEMM
    cudaError_t e = marks.mark(0, st);
    if (e == cudaSuccess && !moe::small_route_permute_ok(*d))  // else the router's kernels clear them
        e = cudaMemsetAsync(hdr, 0, L.clear_bytes, st);          // header + combine counts
    if (e == cudaSuccess) e = route_and_permute(*d, L, x, router_w, router_bias, ws, hdr, marks, st);
    // x quantised once per token, then its codes gathered into expert order
    if (e == cudaSuccess)
        e = moe::launch_quantize_rows(static_cast<const __nv_bfloat16 *>(x), nullptr, 1, d->T, d->H,
                                      at<uint8_t>(ws, L.xq), at<float>(ws, L.xq_s), st);
    if (e == cudaSuccess)
        e = moe::launch_gather_rows_fp8(at<uint8_t>(ws, L.xq), at<float>(ws, L.xq_s), s2f, A, d->H, d->top_k, xs,
                                        xs_s, st);
    if (e == cudaSuccess) e = marks.mark(2, st);
    const int ctas = g_gemm_ctas.load(), rev = g_claim_reverse.load();
    unsigned long long *trace1 = g_trace.load(), *trace2 = trace1 ? trace1 + 2 * g_trace_ctas.load() : nullptr;
    const unsigned long long wl = g_wait_ns.load();
    const uint64_t wait_ns = wl ? wl : 2000000000ull;
    const int stall = g_stall_test.load();
    if (e == cudaSuccess) {
        moe::Fp8GemmArgs g1{0, d->H, d->I, tiles, ntiles, &hdr->counter[0], &hdr->status, xs_s, w_gate_s, w_up_s,
                            h, h_s, nullptr, nullptr, ctas, rev, wait_ns, stall};
        g1.trace = trace1;
        // operands swapped when the groups average at most 64 rows per expert
        const int sw = g_fp8_swap.load();
        const bool swap = sw == 1 || (sw == 0 && moe::tile_choice(A, d->E).fp8_swap_ab);
        e = swap ? moe::launch_grouped_gemm_fp8_swapab(g1, tm_xs, tm_wg, tm_wu, st)
                 : moe::launch_grouped_gemm_fp8(g1, tm_xs, tm_wg, tm_wu, st);
    }
    if (e == cudaSuccess) e = marks.mark(3, st);
    if (e == cudaSuccess) {
        moe::Fp8GemmArgs g2{1, d->I, d->H, tiles, ntiles, &hdr->counter[1], &hdr->status, h_s, w_down_s, w_down_s,
                            nullptr, nullptr, y, s2f, ctas, rev, wait_ns, stall, 0, 1, nullptr, gate,
                            fused ? at<int32_t>(ws, L.ccnt) : nullptr, static_cast<__nv_bfloat16 *>(out), d->top_k,
                            2 * d->top_k};
        g2.trace = trace2;
        e = moe::launch_grouped_gemm_fp8(g2, tm_h, tm_wd, tm_wd, st);
    }
    if (e == cudaSuccess) e = marks.mark(4, st);
    if (e == cudaSuccess && !fused)
        e = moe::launch_combine(y, gate, d->T, d->H, d->top_k, static_cast<__nv_bfloat16 *>(out), st);
    if (e == cudaSuccess) e = marks.mark(5, st);
    return cuda_status(e);
}

moe_status_t moe_quantize_rows_mx(int32_t R, int32_t K, const void *a, uint8_t *q, uint8_t *x, void *stream)
{
    if (R < 0 || K <= 0 || K % 32) return MOE_ERR_INVALID_ARG;
    if (R == 0) return MOE_OK;
    if (!a || !q || !x || !aligned16(a) || !aligned16(q)) return MOE_ERR_INVALID_ARG;
    return cuda_status(moe::launch_quantize_rows_mx(static_cast<const __nv_bfloat16 *>(a), R, K, q, x,
                                                    static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_forward_mx(const moe_dims_t *d, const void *x, const void *router_w, const float *router_bias,
                            const uint8_t *w_gate_p, const uint8_t *w_gate_x, const uint8_t *w_up_p,
                            const uint8_t *w_up_x, const uint8_t *w_down_p, const uint8_t *w_down_x, void *out,
                            void *ws, size_t ws_bytes, void *stream)
{
    moe_status_t s = check_dims(d);
    if (s != MOE_OK) return s;
    if (d->H % 512 || d->I % 512) return MOE_ERR_INVALID_ARG;
    if (d->T == 0) return MOE_OK;
    if (!x || !router_w || !w_gate_p || !w_gate_x || !w_up_p || !w_up_x || !w_down_p || !w_down_x || !out)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(router_w) || !aligned16(w_gate_p) || !aligned16(w_up_p) ||
        !aligned16(w_down_p) || !aligned16(w_gate_x) || !aligned16(w_up_x) || !aligned16(w_down_x) ||
        !aligned16(out))
        return MOE_ERR_INVALID_ARG;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_WORKSPACE;
    const moe::WsLayout L = moe::ws_layout(*d, MOE_DTYPE_MX);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int A = d->T * d->top_k;
    auto *hdr = at<moe::WsHeader>(ws, 0);
    auto *xs = at<uint8_t>(ws, L.xs);
    auto *xs_x = at<uint8_t>(ws, L.xs_s);
    auto *h = at<uint8_t>(ws, L.h);
    auto *h_x = at<uint8_t>(ws, L.h_s);
    auto *y = at<__nv_bfloat16>(ws, L.y);
    auto *gate = at<float>(ws, L.gate);
    auto *s2f = at<int32_t>(ws, L.s2f);
    auto *tiles = at<int32_t>(ws, L.tiles);
    auto *ntiles = at<int32_t>(ws, L.ntiles);

    const int ctas = g_gemm_ctas.load(), rev = g_claim_reverse.load();
    unsigned long long *trace1 = g_trace.load(), *trace2 = trace1 ? trace1 + 2 * g_trace_ctas.load() : nullptr;
    const unsigned long long wl = g_wait_ns.load();
    const uint64_t wait_ns = wl ? wl : 2000000000ull;
    const int stall = g_stall_test.load();
    moe::MxLaunch g1{0, d->H, d->I, tiles, ntiles, &hdr->counter[0], &hdr->status, h, h_x, nullptr, nullptr,
                     ctas, rev, wait_ns, stall, trace1};
    moe::MxLaunch g2{1, d->I, d->H, tiles, ntiles, &hdr->counter[1], &hdr->status, nullptr, nullptr, y, s2f,
                     ctas, rev, wait_ns, stall, trace2};
    if (!moe::encode_a_maps(&g1.tmX, xs, A, d->H, true) ||
        !encode_4d_fp4_pairs(&g1.tmW0, w_gate_p, d->E, d->I, d->H, 128) ||
        !encode_4d_fp4_pairs(&g1.tmW1, w_up_p, d->E, d->I, d->H, 128) ||
        !encode_scales_u8(&g1.tmSX, xs_x, 1, A, d->H / 32, 64, 2) ||
        !encode_scales_u8(&g1.tmSW0, w_gate_x, d->E, d->I, d->H / 32, 128, 3) ||
        !encode_scales_u8(&g1.tmSW1, w_up_x, d->E, d->I, d->H / 32, 128, 3) ||
        !moe::encode_a_maps(&g2.tmX, h, A, d->I, true) ||
        !encode_4d_fp4_pairs(&g2.tmW0, w_down_p, d->E, d->H, d->I, 128) ||
        !encode_scales_u8(&g2.tmSX, h_x, 1, A, d->I / 32, 64, 2) ||
        !encode_scales_u8(&g2.tmSW0, w_down_x, d->E, d->H, d->I / 32, 128, 3))
        return MOE_ERR_CUDA;
    g2.tmW1 = g2.tmW0;    // the down GEMM's two tiles are rows n0.. and n0+128.. of w_down
    g2.tmSW1 = g2.tmSW0;

    const StageMarks marks;
    cudaError_t e = marks.mark(0, st);
    if (e == cudaSuccess && !moe::small_route_permute_ok(*d))  // else the router's kernels clear them
        e = cudaMemsetAsync(hdr, 0, L.clear_bytes, st);
    if (e == cudaSuccess) e = route_and_permute(*d, L, x, router_w, router_bias, ws, hdr, marks, st);
    // x quantised once per token, then its codes and scale codes gathered into expert order
    if (e == cudaSuccess)
        e = moe::launch_quantize_rows_mx(static_cast<const __nv_bfloat16 *>(x), d->T, d->H, at<uint8_t>(ws, L.xq),
                                         at<uint8_t>(ws, L.xq_s), st);
    if (e == cudaSuccess)
        e = moe::launch_gather_rows_mx(at<uint8_t>(ws, L.xq), at<uint8_t>(ws, L.xq_s), s2f, A, d->H, d->top_k, xs,
                                       xs_x, st);
    if (e == cudaSuccess) e = marks.mark(2, st);
    if (e == cudaSuccess) e = moe::launch_grouped_gemm_mx(g1, st);
    if (e == cudaSuccess) e = marks.mark(3, st);
    if (e == cudaSuccess) e = moe::launch_grouped_gemm_mx(g2, st);
    if (e == cudaSuccess) e = marks.mark(4, st);
    if (e == cudaSuccess) e = moe::launch_combine(y, gate, d->T, d->H, d->top_k, static_cast<__nv_bfloat16 *>(out), st);
    if (e == cudaSuccess) e = marks.mark(5, st);
    return cuda_status(e);
}

int32_t moe_forward_plan(const moe_dims_t *d, int dtype)
{
    if (moe_workspace_size(d, dtype) == 0) return -1;
    if (dtype != MOE_DTYPE_BF16) {  // the fp8 and MX forwards: small router, fused combine for fp8
        const bool fused = dtype == MOE_DTYPE_FP8 && d->T <= moe::kFusedCombineMaxTFp8;
        return (moe::small_route_permute_ok(*d) ? MOE_PLAN_SMALL_ROUTER : 0) | (fused ? MOE_PLAN_FUSED_COMBINE : 0);
    }
    return bf16_plan(*d);
}

moe_status_t moe_workspace_offsets(const moe_dims_t *d, int dtype, size_t *out, int32_t n)
{
    if (!out || n < 0 || moe_workspace_size(d, dtype) == 0) return MOE_ERR_INVALID_ARG;
    const moe::WsLayout L = moe::ws_layout(*d, dtype);
    const size_t v[13] = {L.idx, L.gate, L.offsets, L.s2f, L.f2s, L.tiles, L.ntiles, L.logits,
                          L.xs, L.xs_s, L.h, L.h_s, L.y};
    for (int i = 0; i < n && i < 13; ++i) out[i] = v[i];
    return MOE_OK;
}

moe_status_t moe_get_device_status(void *ws, void *stream)
{
    if (!ws) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
    int32_t v = 0;
    if (cudaMemcpy(&v, ws, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
    const int32_t zero = 0;
    if (cudaMemcpy(ws, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess) return MOE_ERR_CUDA;
    return static_cast<moe_status_t>(v);
}

}  // extern "C"
