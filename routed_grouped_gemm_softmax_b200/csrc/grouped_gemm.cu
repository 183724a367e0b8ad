// grouped_gemm.cu -- persistent grouped GEMMs of the expert FFN on the 5th-gen
// tensor cores (tcgen05 + TMEM + TMA), sm_100a.
//
// Work decomposition.  The expert FFN is a batch of small GEMMs, one per expert
// group (GC-MoE page: "grouped GEMM batches the experts' small matrix products
// into one kernel"; vLLM fused-MoE page, section 02).  A work item is one
// (m-tile, n-tile) pair, where the m-tiles are the 128-row blocks of the expert
// groups listed by the permutation (FlashMoE, section 3: 128x128-class tile
// tasks).  CTAs are persistent -- one per SM -- and claim the next item from a
// global atomic counter whenever they are free (the Weave review, section 2.2:
// a task queue plus an atomic counter from which idle SMs grab the next task),
// so a hot expert's many tiles spread over every SM instead of queueing on a
// fixed subset.  Items are numbered m-tile-major, so the n-tiles of one m-tile
// and the m-tiles of one expert are claimed close together and share the A rows
// and the expert's weight tiles in L2 (the GROUP_SIZE_M idea of the vLLM page,
// section 03).
//
// CTA roles (192 threads):
//   warp 0, lane 0: claims items, feeds a ring of item ids to the other roles,
//                   and streams A and B tiles into a 4-stage shared-memory ring
//                   with TMA (128-byte swizzle), one mbarrier pair per stage;
//                   with direct A rows, the 32 lanes each gather four x rows of
//                   a gate/up tile per stage (tile::gather4), so no expert-ordered
//                   copy of x is written;
//   warp 1        : allocates 512 TMEM columns; lane 0 issues tcgen05.mma
//                   (M=128, N=256, K=16, bf16 in, fp32 accumulate) into one of
//                   two TMEM accumulators, releasing each stage with
//                   tcgen05.commit;
//   warps 2-5     : epilogue -- tcgen05.ld of the accumulator (each warp reads
//                   its 32-lane quarter), then
//                   mode 0 (gate/up): h = silu(gate) * up, rounded to bf16,
//                   mode 1 (down)   : y row of the assignment, rounded to bf16,
//                                     then the fused combine (combine.cuh),
//                   mode 2 (dense)  : fp32 rows (the router's tensor-core logits),
//                   rows past the group's end masked.
// Every accumulation order is fixed by the tile and the K loop, never by which
// CTA ran the item, so results are bitwise independent of the schedule.
// Every wait is bounded (GemmArgs::wait_ns); a wait that runs out records
// MOE_ERR_TIMEOUT in the workspace status word and the CTA unwinds -- waiting,
// with the fixed default bound, for its own TMA copies and MMAs -- before
// freeing TMEM.
#include <mutex>

#include "combine.cuh"
#include "moe_internal.h"
#include "pdl.cuh"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

constexpr int BM = kTileRows;  // 128 rows per tile
constexpr int BK = 64;         // a K chunk: 64 bf16 = one 128-byte swizzle row
constexpr int KC = 2;          // K chunks per stage
constexpr int BKS = BK * KC;   // K of a stage: 128
constexpr int BN = 256;        // output columns per item (gate/up: 128 + 128)
// Two stages of 128 K columns (96 KB) rather than four of 64: each weight box then
// brings both chunks of its rows, 256 contiguous bytes a row, which DRAM streams about
// a third faster than 128-byte row pieces, and fewer bytes wait on more barriers.
constexpr int STAGES = 2;
constexpr int RING = 4;
constexpr int A_SUB = BM * BK * 2;     // 16 KB: one chunk of A rows
constexpr int B_SUB = BN * BK * 2;     // 32 KB: one chunk of B rows
constexpr int A_BYTES = A_SUB * KC;    // 32 KB
constexpr int B_BYTES = B_SUB * KC;    // 64 KB
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;   // two 128 x 256 fp32 accumulators

struct Ctrl {
    uint64_t full[STAGES];   // TMA bytes landed in stage s
    uint64_t empty[STAGES];  // MMAs reading stage s finished
    uint64_t accf[2];        // accumulator a holds a finished tile
    uint64_t acce[2];        // epilogue drained accumulator a
    uint64_t itf[RING];      // ring slot r holds the next item id
    uint64_t ite[RING];      // every role has read ring slot r
    uint64_t fin;            // all MMAs of this CTA are done
    uint64_t never;          // nothing ever arrives here (timeout test)
    int32_t ring[RING];
    uint32_t tmem_base;
};

constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * (A_BYTES + B_BYTES) + sizeof(Ctrl);

__device__ __forceinline__ void record_status(int32_t *status, int code) { atomicCAS(status, 0, code); }

__device__ __forceinline__ float silu(float a) { return a / (1.0f + __expf(-a)); }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Item `item` of the launch: its phase (1: a down item; in modes 0-2 fixed by the
// mode, in mode 3 the items past the gate/up ones), m-tile and n-tile.
struct ItemPos {
    int p1, mt, nt;
};

// Waits (at most limit_ns) until *ctr >= target, with acquire ordering at GPU scope.
__device__ __forceinline__ bool wait_count_at_least(const int32_t *ctr, int target, uint64_t limit_ns)
{
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
    if (v >= target) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i) {
            asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
            if (v >= target) return true;
        }
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
}

__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

template <int MODE>
__global__ void __launch_bounds__(THREADS, 1)
grouped_gemm_kernel(const __grid_constant__ AMaps tmA, const __grid_constant__ CUtensorMap tmB0,
                    const __grid_constant__ CUtensorMap tmB1, const GemmArgs g, const __grid_constant__ SharedMaps sm,
                    const __grid_constant__ LayerMaps lm)
{
    // Output columns per tile: the gate/up items pack 128 gate + 128 up columns into
    // N=256; the down (and dense) items write 256 columns.
    constexpr int BNO0 = BN / 2, BNO1 = BN;
    const bool dense = g.tiles == nullptr;  // mode 2: m-tiles are plain 128-row blocks of A
    extern __shared__ uint8_t smem_raw[];
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    uint8_t *sA = smem_raw + pad;
    uint8_t *sB = sA + STAGES * A_BYTES;
    Ctrl *S = reinterpret_cast<Ctrl *>(sB + STAGES * B_BYTES);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    // n-tiles and K blocks of the gate/up items (modes 0, 3) and of the down / dense items
    const int nt0 = (g.N + BNO0 - 1) / BNO0, kb0 = (g.K + BKS - 1) / BKS;
    const int nt1 = MODE == 3 ? (g.N2 + BNO1 - 1) / BNO1 : (g.N + BNO1 - 1) / BNO1;
    const int K1 = MODE == 3 ? g.K2 : g.K;  // K of the down (or dense) items
    const int kb1 = (K1 + BKS - 1) / BKS;
    // K chunks of stage kb of a K range of Kd columns (a multiple of 64)
    auto chunks_of = [](int kb, int Kd) { return min(KC, (Kd - kb * BKS) / BK); };

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&S->full[s], 1);
            mbar_init(&S->empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&S->accf[a], 1);
            mbar_init(&S->acce[a], 4);
        }
        for (int r = 0; r < RING; ++r) {
            mbar_init(&S->itf[r], 1);
            mbar_init(&S->ite[r], 5);  // the MMA thread + 4 epilogue warps
        }
        mbar_init(&S->fin, 1);
        mbar_init(&S->never, 1);
        fence_mbar_init();
        for (int b = 0; b < kABoxes; ++b) tma_prefetch_desc(&tmA.m[b]);
        tma_prefetch_desc(&tmB0);
        if (MODE == 0 || MODE == 3) tma_prefetch_desc(&tmB1);
        if (MODE == 3) tma_prefetch_desc(&lm.wd);
        if (g.sh_count) {
            tma_prefetch_desc(&sm.b0);
            if (MODE == 0 || MODE == 3) tma_prefetch_desc(&sm.b1);
        }
        if ((MODE == 0 || MODE == 3) && g.a_rows) tma_prefetch_desc(&sm.xg);
    }
    if (warp == 1) tmem_alloc(&S->tmem_base, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S->tmem_base;
    // The prologue above overlapped the previous kernel.  Modes 0, 1 and 3: warp 0
    // waits for it inside the producer, after the first stages' weight loads (the
    // weights are the layer's inputs; only the A rows are the previous kernel's output).
    // (GemmArgs::tiles_first: the tile list itself is the previous kernel's output, so
    // warp 0 waits first.)
    const bool early_b = MODE != 2 && !g.tiles_first;
    if (!(early_b && warp == 0)) pdl_wait();
    pdl_trigger();
    if (g.trace && threadIdx.x == 0) g.trace[2 * blockIdx.x] = globaltimer_ns();

    // m-tiles: the tile list's, then the shared expert's; the gate/up items of all
    // m-tiles precede (mode 3) the down items
    const int nrouted = dense ? 0 : *g.ntiles;
    const int sh_tps = g.sh_count ? (g.sh_T + BM - 1) / BM : 1;
    const int mtiles = dense ? (g.M + BM - 1) / BM : nrouted + g.sh_count * sh_tps;
    const int total0 = MODE == 3 ? mtiles * nt0 : 0;
    auto pos_of = [&](int item) {
        ItemPos r;
        r.p1 = MODE == 1 || MODE == 2 || (MODE == 3 && item >= total0);
        const int local = MODE == 3 && r.p1 ? item - total0 : item;
        const int ntl = r.p1 ? nt1 : nt0;
        r.mt = local / ntl;
        r.nt = local - r.mt * ntl;
        return r;
    };

    if (warp == 0) {
        // ------------------------------------------------ scheduler + TMA producer
        // Lane 0 claims the items, keeps the rings and loads B (and A with row-block
        // boxes); with direct A rows (GemmArgs::a_rows) each lane gathers four A rows of a
        // routed gate/up tile per stage, lane l rows 4l..4l+3.
        const bool gather = (MODE == 0 || MODE == 3) && g.a_rows != nullptr;
        const int total = MODE == 3 ? total0 + mtiles * nt1 : mtiles * (MODE == 0 ? nt0 : nt1);
        int stage = 0, rs = 0;
        uint32_t phase = 0, rphase = 0;
        uint32_t armed = 0, armed_par = 0;  // stages with a load issued, and its phase
        bool ok = true;
        int cursor = (int)blockIdx.x * (g.reverse == 2);  // static modes
        bool held = early_b;  // A loads of the first item's first stages wait for the previous kernel
        for (;;) {
            int item = -1, okl = 1;
            if (lane == 0) {
                if (MODE != 3) {
                    item = claim_item(g.reverse, g.counter, total, MODE == 0 ? nt0 : nt1, dense ? nullptr : g.tiles,
                                      cursor, nrouted, g.sh_e0, sh_tps);
                } else if (g.reverse <= 1) {
                    // the queue; descending within each phase, so that every gate/up item is
                    // claimed before any down item whatever the order
                    item = atomicAdd(g.counter, 1);
                    if (item >= total) item = -1;
                    else if (g.reverse == 1)
                        item = item < total0 ? total0 - 1 - item : total0 + (total - 1 - item);
                } else {
                    // static: this CTA's items in ascending order, every c-th (mode 2) or those
                    // of the experts e with e % grid == c (mode 3)
                    while (cursor < total) {
                        const int it = cursor;
                        cursor += g.reverse == 2 ? (int)gridDim.x : 1;
                        if (g.reverse == 2) { item = it; break; }
                        const TileRef t = tile_ref(g.tiles, nrouted, pos_of(it).mt, BM, 0, g.sh_T, g.sh_rows0, g.sh_e0);
                        if (t.e % (int)gridDim.x == (int)blockIdx.x) { item = it; break; }
                    }
                }
                if (mbar_wait(&S->ite[rs], rphase ^ 1, g.wait_ns)) {
                    S->ring[rs] = item;
                    mbar_arrive(&S->itf[rs]);
                } else {
                    okl = 0;
                }
            }
            item = __shfl_sync(0xffffffffu, item, 0);
            if (!__shfl_sync(0xffffffffu, okl, 0)) { ok = false; break; }
            if (++rs == RING) { rs = 0; rphase ^= 1; }
            if (item < 0) break;
            const ItemPos ip = pos_of(item);
            const bool p1 = ip.p1;
            TileRef tr{0, ip.mt * BM, 0, ip.mt * BM, -1};
            if (dense)
                tr.rows = min(BM, g.M - tr.row0);
            else
                tr = tile_ref(g.tiles, nrouted, ip.mt, BM, p1 ? 1 : 0, g.sh_T, g.sh_rows0, g.sh_e0);
            const int expert = tr.e, arow0 = tr.arow0;
            const int ab = a_box(tr.rows);  // the A box that covers the tile's rows
            const CUtensorMap *amap = MODE == 3 && p1 ? &lm.h.m[ab]
                                    : (!p1 && tr.s >= 0) ? &sm.x.m[ab] : &tmA.m[ab];
            // direct rows: the x rows (tokens) of this lane's four tile rows, the tail's
            // missing rows repeating the tile's last one (their products are masked)
            const bool g4 = gather && !p1 && tr.s < 0;
            const bool g4_lane = g4 && 4 * lane < tr.rows;
            int tok[4] = {0, 0, 0, 0};
            auto load_tokens = [&]() {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int t = g.a_rows[tr.row0 + min(4 * lane + j, tr.rows - 1)] / g.a_div;
                    tok[j] = (unsigned)t < (unsigned)g.a_tokens ? t : 0;
                }
            };
            if (g4_lane && !held) load_tokens();
            // per K chunk; the weight boxes bring all KC chunks of their rows (a chunk past
            // the K range reads zeros and is not multiplied)
            const uint32_t a_bytes = g4 ? (uint32_t)((tr.rows + 3) / 4) * 512u : (uint32_t)(a_box_rows(ab) * BK * 2);
            const int n0 = ip.nt * (p1 ? BNO1 : BNO0);
            const int num_kb = p1 ? kb1 : kb0;
            const int Kd = p1 ? K1 : g.K;
            if (MODE == 3 && p1) {
                // the down item reads h rows of m-tile mt: wait until every gate/up item of
                // mt has published them, then order those generic-proxy writes before the
                // TMA (async-proxy) reads below
                if (lane == 0) {
                    okl = wait_count_at_least(g.ready + ip.mt, 4 * nt0, g.wait_ns);
                    fence_proxy_async_global();
                }
                if (!__shfl_sync(0xffffffffu, okl, 0)) { ok = false; break; }
            }
            for (int kb = 0; kb < num_kb; ++kb) {
                const int nc = chunks_of(kb, Kd);
                if (lane == 0) {
                    okl = mbar_wait(&S->empty[stage], phase ^ 1, g.wait_ns);
                    if (okl) {
                        mbar_arrive_expect_tx(&S->full[stage], a_bytes * nc + B_BYTES);
                        armed |= 1u << stage;
                        armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
                        uint8_t *b_dst = sB + stage * B_BYTES;
                        const int z = kb * KC;  // first K chunk of the stage
                        if (!held && !g4)
                            for (int c = 0; c < nc; ++c)
                                tma_load_2d(sA + stage * A_BYTES + c * A_SUB, amap, &S->full[stage], (z + c) * BK, arow0);
                        if (!p1) {  // gate / up rows n0.. of the expert (or of shared slice s): [KC][128] each
                            if (tr.s < 0) {
                                tma_load_4d(b_dst, &tmB0, &S->full[stage], 0, n0, z, expert);
                                tma_load_4d(b_dst + B_BYTES / 2, &tmB1, &S->full[stage], 0, n0, z, expert);
                            } else {
                                tma_load_3d(b_dst, &sm.b0, &S->full[stage], 0, tr.s * g.N + n0, z);
                                tma_load_3d(b_dst + B_BYTES / 2, &sm.b1, &S->full[stage], 0, tr.s * g.N + n0, z);
                            }
                        } else {  // down rows n0..: the expert's, or chunks of columns s*I.. of the shared down: [KC][256]
                            const CUtensorMap *bm = MODE == 3 ? &lm.wd : &tmB0;
                            const CUtensorMap *bs = MODE == 3 ? &lm.wd_sh : &sm.b0;
                            if (tr.s < 0)
                                tma_load_4d(b_dst, bm, &S->full[stage], 0, n0, z, expert);
                            else
                                tma_load_3d(b_dst, bs, &S->full[stage], 0, n0, tr.s * (K1 / BK) + z);
                        }
                    }
                }
                if (!__shfl_sync(0xffffffffu, okl, 0)) { ok = false; break; }
                if (g4_lane && !held)
                    for (int c = 0; c < nc; ++c)
                        tma_gather4(sA + stage * A_BYTES + c * A_SUB + lane * 512, &sm.xg, &S->full[stage],
                                    (kb * KC + c) * BK, tok[0], tok[1], tok[2], tok[3]);
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
                if (held && kb + 1 == min(STAGES, num_kb)) {  // first item: stage j holds K block j
                    pdl_wait();
                    held = false;
                    if (g4_lane) load_tokens();
                    for (int j = 0; j <= kb; ++j)
                        for (int c = 0; c < chunks_of(j, Kd); ++c) {
                            if (g4_lane)
                                tma_gather4(sA + j * A_BYTES + c * A_SUB + lane * 512, &sm.xg, &S->full[j],
                                            (j * KC + c) * BK, tok[0], tok[1], tok[2], tok[3]);
                            else if (!g4 && lane == 0)
                                tma_load_2d(sA + j * A_BYTES + c * A_SUB, amap, &S->full[j], (j * KC + c) * BK, arow0);
                        }
                }
            }
            if (!ok) break;
        }
        if (lane == 0) {
            if (!ok) {
                record_status(g.status, MOE_ERR_TIMEOUT);
                if (mbar_wait(&S->ite[rs], rphase ^ 1)) {
                    S->ring[rs] = -1;
                    mbar_arrive(&S->itf[rs]);
                }
            }
            // never leave with TMA copies still landing in shared memory
            for (int s = 0; s < STAGES; ++s)
                if ((armed >> s) & 1u)
                    if (!mbar_wait(&S->full[s], (armed_par >> s) & 1u)) record_status(g.status, MOE_ERR_TIMEOUT);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN);           // down: N = 256
            constexpr uint32_t IDESC_H = idesc_bf16_f32(BM, BN / 2);     // gate, up: N = 128 each
            int stage = 0, rs = 0, acc = 0;
            uint32_t phase = 0, rphase = 0, aphase = 0;
            // timeout test: wait (bounded) on a barrier nothing signals, then unwind
            bool ok = !(g.stall_test && !mbar_wait(&S->never, 0, g.wait_ns));
            while (ok) {
                if (!mbar_wait(&S->itf[rs], rphase, g.wait_ns)) { ok = false; break; }
                const int item = S->ring[rs];
                mbar_arrive(&S->ite[rs]);
                if (++rs == RING) { rs = 0; rphase ^= 1; }
                if (item < 0) break;
                const bool p1 = pos_of(item).p1;
                const int num_kb = p1 ? kb1 : kb0, Kd = p1 ? K1 : g.K;
                if (!mbar_wait(&S->acce[acc], aphase ^ 1, g.wait_ns)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d = tmem + static_cast<uint32_t>(acc * BN);
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(&S->full[stage], phase, g.wait_ns)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sA + stage * A_BYTES);
                    const uint32_t b0 = smem_u32(sB + stage * B_BYTES);
                    const int nc = chunks_of(kb, Kd);
                    for (int c = 0; c < nc; ++c) {
                        const uint32_t ac = a0 + c * A_SUB;
                        if (!p1) {
                            // gate rows [KC][128] then up rows [KC][128]: an N = 128 MMA into
                            // each half of the accumulator (gate columns 0..127, up 128..255)
                            const uint32_t bg = b0 + c * (B_SUB / 2), bu = b0 + B_BYTES / 2 + c * (B_SUB / 2);
#pragma unroll
                            for (int k = 0; k < BK / 16; ++k) {
                                const uint64_t ad = sw128_kmajor_desc(ac + k * 32);
                                mma_bf16(d, ad, sw128_kmajor_desc(bg + k * 32), IDESC_H, (kb | c | k) != 0);
                                mma_bf16(d + BN / 2, ad, sw128_kmajor_desc(bu + k * 32), IDESC_H, (kb | c | k) != 0);
                            }
                        } else {
                            const uint32_t bc = b0 + c * B_SUB;
#pragma unroll
                            for (int k = 0; k < BK / 16; ++k)
                                mma_bf16(d, sw128_kmajor_desc(ac + k * 32), sw128_kmajor_desc(bc + k * 32), IDESC,
                                         (kb | c | k) != 0);
                        }
                    }
                    mma_commit(&S->empty[stage]);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                mma_commit(&S->accf[acc]);
                if (++acc == 2) { acc = 0; aphase ^= 1; }
            }
            if (!ok) record_status(g.status, MOE_ERR_TIMEOUT);
            // TMEM may only be released once every MMA issued here has completed
            mma_commit(&S->fin);
            if (!mbar_wait(&S->fin, 0)) record_status(g.status, MOE_ERR_TIMEOUT);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;  // TMEM lane quarter this warp may read
        const int row = q * 32 + lane;
        int rs = 0, acc = 0;
        uint32_t rphase = 0, aphase = 0;
        // y row of sorted row r: the row map's for the routed rows, r itself for the shared expert's
        auto flat_of = [&](int r) { return (g.sh_count == 0 || r < g.sh_rows0) ? g.row_map[r] : r; };
        for (;;) {
            if (!mbar_wait(&S->itf[rs], rphase, g.wait_ns)) { record_status(g.status, MOE_ERR_TIMEOUT); break; }
            const int item = S->ring[rs];
            __syncwarp();
            if (lane == 0) mbar_arrive(&S->ite[rs]);
            if (++rs == RING) { rs = 0; rphase ^= 1; }
            if (item < 0) break;
            const ItemPos ip = pos_of(item);
            const bool p1 = ip.p1;
            const int nt = ip.nt;
            int row0 = ip.mt * BM, rows = 0;
            if (dense) {
                rows = min(BM, g.M - row0);
            } else {
                const TileRef tr = tile_ref(g.tiles, nrouted, ip.mt, BM, p1 ? 1 : 0, g.sh_T, g.sh_rows0, g.sh_e0);
                row0 = tr.row0;
                rows = tr.rows;
            }
            const bool row_ok = row < rows;
            if (!mbar_wait(&S->accf[acc], aphase, g.wait_ns)) { record_status(g.status, MOE_ERR_TIMEOUT); break; }
            tc_fence_after();
            const uint32_t tb = tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * BN);
            if (!p1) {
                __nv_bfloat16 *orow = g.out + (size_t)(row0 + row) * g.N;
#pragma unroll 1
                for (int c = 0; c < BNO0 / 32; ++c) {
                    uint32_t gr[32], ur[32];
                    tmem_ld32_sync(tb + c * 32, gr);
                    tmem_ld32_sync(tb + BNO0 + c * 32, ur);
                    const int col = nt * BNO0 + c * 32;
                    if (row_ok && col < g.N) {
                        uint32_t pk[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const float h0 = silu(__uint_as_float(gr[2 * i])) * __uint_as_float(ur[2 * i]);
                            const float h1 = silu(__uint_as_float(gr[2 * i + 1])) * __uint_as_float(ur[2 * i + 1]);
                            pk[i] = pack_bf16(h0, h1);
                        }
                        uint4 *dst = reinterpret_cast<uint4 *>(orow + col);
#pragma unroll
                        for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                    }
                }
            } else if (MODE == 2) {
                float *orow = g.out_f32 + (size_t)(row0 + row) * g.N;
#pragma unroll 1
                for (int c = 0; c < BNO1 / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32_sync(tb + c * 32, r);
                    const int col = nt * BNO1 + c * 32;
                    if (row_ok && col + 32 <= g.N && (g.N & 3) == 0) {  // rows 16-byte aligned
                        float4 *dst = reinterpret_cast<float4 *>(orow + col);
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            dst[i] = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                                 __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
                    } else if (row_ok && col < g.N) {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (col + i < g.N) orow[col + i] = __uint_as_float(r[i]);
                    }
                }
            } else {
                const int N = MODE == 3 ? g.N2 : g.N;
                __nv_bfloat16 *y = MODE == 3 ? g.out2 : g.out;
                const int flat = row_ok ? flat_of(row0 + row) : 0;
                __nv_bfloat16 *orow = y + (size_t)flat * N;
#pragma unroll 1
                for (int c = 0; c < BNO1 / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32_sync(tb + c * 32, r);
                    const int col = nt * BNO1 + c * 32;
                    if (row_ok && col < N) {
                        uint32_t pk[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) pk[i] = pack_bf16(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
                        uint4 *dst = reinterpret_cast<uint4 *>(orow + col);
#pragma unroll
                        for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S->acce[acc]);
            if (++acc == 2) { acc = 0; aphase ^= 1; }
            if (MODE == 3 && !p1) {
                // publish this warp's h rows of m-tile mt to the down items: each lane's
                // stores before the warp's count (release at GPU scope), visible to the TMA
                // reads that follow the consumer's acquire
                fence_proxy_async_global();
                __syncwarp();
                if (lane == 0) {
                    __threadfence();
                    atomicAdd(g.ready + ip.mt, 1);
                }
            }
            if ((MODE == 1 || (MODE == 3 && p1)) && g.comb_cnt)  // the accumulator is already released
                combine_arrive(MODE == 3 ? g.out2 : g.out, g.comb_gate, g.comb_out, g.comb_cnt, g.comb_k,
                               g.comb_target, MODE == 3 ? g.N2 : g.N, nt1, nt, row_ok,
                               row_ok ? flat_of(row0 + row) : 0, lane, g.sh_count, g.sh_T, g.sh_rows0);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (g.trace && threadIdx.x == 0) g.trace[2 * blockIdx.x + 1] = globaltimer_ns();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace

int num_sms()
{
    static int cached[64] = {};
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    if (dev >= 0 && dev < 64) cached[dev] = n;
    return n;
}

// The kernels need more than the default 48 KB of dynamic shared memory; the
// attribute is set once per device (and per kernel) rather than on every launch.
static bool smem_attr_ready(int mode)
{
    static std::mutex mu;
    static uint64_t done[4] = {0, 0, 0, 0};  // bit per device
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    std::lock_guard<std::mutex> lk(mu);
    if (done[mode] >> dev & 1ull) return true;
    const int a = (int)SMEM_BYTES;
    if (mode == 2) return false;  // no dense mode: the router's tensor-core logits run in the fp8 kernel
    cudaError_t e = mode == 0   ? cudaFuncSetAttribute(grouped_gemm_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, a)
                  : mode == 1 ? cudaFuncSetAttribute(grouped_gemm_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, a)
                              : cudaFuncSetAttribute(grouped_gemm_kernel<3>, cudaFuncAttributeMaxDynamicSharedMemorySize, a);
    if (e != cudaSuccess) return false;
    done[mode] |= 1ull << dev;
    return true;
}

cudaError_t launch_grouped_gemm(const GemmArgs &g, const AMaps &tmA, const CUtensorMap &tmB0,
                                const CUtensorMap &tmB1, cudaStream_t st, const SharedMaps *sm, const LayerMaps *lm)
{
    const int grid = g.ctas > 0 ? g.ctas : num_sms();
    if (g.mode < 0 || g.mode > 3 || g.mode == 2 || !smem_attr_ready(g.mode)) return cudaErrorInvalidValue;
    if (g.sh_count && (!sm || g.mode == 2)) return cudaErrorInvalidValue;
    if (g.mode == 3 && (!lm || !g.ready)) return cudaErrorInvalidValue;
    if (g.a_rows && (!sm || g.a_div <= 0 || g.a_tokens <= 0 || (g.mode != 0 && g.mode != 3))) return cudaErrorInvalidValue;
    static const SharedMaps none{};
    static const LayerMaps nolm{};
    const SharedMaps &s = sm ? *sm : none;
    const LayerMaps &l = lm ? *lm : nolm;
    switch (g.mode) {
    case 0: return launch_pdl(grouped_gemm_kernel<0>, dim3(grid), dim3(THREADS), SMEM_BYTES, st, tmA, tmB0, tmB1, g, s, l);
    case 1: return launch_pdl(grouped_gemm_kernel<1>, dim3(grid), dim3(THREADS), SMEM_BYTES, st, tmA, tmB0, tmB1, g, s, l);
    default: return launch_pdl(grouped_gemm_kernel<3>, dim3(grid), dim3(THREADS), SMEM_BYTES, st, tmA, tmB0, tmB1, g, s, l);
    }
}

}  // namespace moe
