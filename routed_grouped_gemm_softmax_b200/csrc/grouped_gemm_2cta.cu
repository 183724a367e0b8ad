// grouped_gemm_2cta.cu -- the bf16 grouped GEMMs with pair-of-CTA MMAs
// (tcgen05 cta_group::2), for expert groups large enough to be compute-bound.
//
// A work item is one (pair tile, n-tile): a pair tile is up to 256 rows of one
// expert group, split 128 + 128 over the two CTAs of a cluster.  One MMA of
// M = 256, N = 256, K = 16 reads the A rows from both CTAs' shared memory and B
// from both too -- each CTA holds only half of the 256 B rows (the gate rows on
// CTA 0 and the up rows on CTA 1 in the gate/up GEMM; the first and second 128
// output columns in the down GEMM) -- so per CTA a 64-wide K block moves 32 KB
// instead of the 48 KB of the one-CTA kernel for the same tensor-core work.  Each
// CTA's TMEM accumulator holds its own 128 rows x 256 columns, so the epilogue is
// the one-CTA kernel's.
//
// Roles: CTA 0 (the leader) claims items from the atomic queue and hands each one
// to CTA 1 through its shared memory; in both CTAs warp 0 streams that CTA's A and
// B halves with TMA, completing on the leader's stage barrier (with direct A rows the
// warp's 32 lanes gather a gate/up tile's x rows four at a time, tile::gather4, so
// no expert-ordered copy of x is written); the leader's warp 1
// issues the MMAs and commits each stage, the accumulators and the end to both
// CTAs' barriers at once (tcgen05.commit with a CTA mask); warps 2-5 of both CTAs
// drain their accumulator halves.  No TMA load is multicast.  Every wait is
// bounded, and a CTA leaves only after the other has finished touching it.
#include <mutex>

#include "combine.cuh"
#include "moe_internal.h"
#include "pdl.cuh"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

constexpr int HALF = kTileRows;        // rows per CTA of a pair tile
constexpr int BK2 = 64;                // one TMA box: 64 bf16 = one 128-byte swizzle row
constexpr int KW2 = 2;                 // 64-column boxes per stage
constexpr int BKS2 = BK2 * KW2;        // K of a stage: 128
constexpr int BN2 = 256;               // MMA N (128 B rows per CTA)
// Three stages of 64 KB rather than six of 32 KB: a stage's loads complete on one
// barrier, and the SM's TMA throughput from L2 grows with the bytes behind each
// barrier (about 71 GB/s per SM with two 16 KB boxes per stage, 109 GB/s with four).
constexpr int ST2 = 3;
constexpr int RING2 = 4;
constexpr int A2_SUB = HALF * BK2 * 2;     // 16 KB: one box of A rows
constexpr int B2_SUB = 128 * BK2 * 2;      // 16 KB: one box of B rows
constexpr int A2_BYTES = A2_SUB * KW2;     // 32 KB
constexpr int B2_BYTES = B2_SUB * KW2;     // 32 KB
constexpr int THREADS2 = 192;
constexpr uint32_t TMEM_COLS2 = 512;

struct Ctrl2 {
    uint64_t full[ST2];    // leader: both CTAs' TMA bytes of stage s landed (2 arrivals + tx)
    uint64_t empty[ST2];   // each: the pair's MMAs reading stage s finished
    uint64_t accf[2];      // each: accumulator a holds a finished tile
    uint64_t acce[2];      // leader: all 8 epilogue warps drained accumulator a
    uint64_t itf[RING2];   // each: ring slot r holds the next item
    uint64_t ite[RING2];   // leader: the 10 consumers of both CTAs read slot r
    uint64_t fin;          // each: every MMA of the pair completed
    uint64_t bye;          // each: the other CTA is done touching this one
    int32_t ring[RING2];
    uint32_t tmem_base;
};

constexpr size_t SMEM2 = 1024 + (size_t)ST2 * (A2_BYTES + B2_BYTES) + sizeof(Ctrl2);

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t peer_addr(const void *p, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
    return r;
}
__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void arrive_remote(uint32_t bar)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar) : "memory");
}
// The stage arrival of the peer's producer: relaxed, since it publishes no data of
// its own (its TMA bytes complete on the barrier themselves); a release at cluster
// scope would wait for every earlier memory operation of the thread.
__device__ __forceinline__ void arrive_expect_tx_remote(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.relaxed.cluster.shared::cluster.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void st_remote(uint32_t addr, int32_t v)
{
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
// TMA tile loads into this CTA's shared memory that complete on a barrier of either CTA.
__device__ __forceinline__ void tma_load_2d_pair(void *dst, const CUtensorMap *tm, uint32_t bar, int x, int y)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(bar), "r"(x), "r"(y)
        : "memory");
}
// Four rows r0..r3 of a one-row-box tensor map to this CTA's dst, signalling the
// leader CTA's barrier (tile::gather4 of a CTA pair).
__device__ __forceinline__ void tma_gather4_pair(void *dst, const CUtensorMap *tm, uint32_t bar, int x, int r0, int r1,
                                                 int r2, int r3)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(bar), "r"(x), "r"(r0), "r"(r1), "r"(r2), "r"(r3)
        : "memory");
}
__device__ __forceinline__ void tma_load_4d_pair(void *dst, const CUtensorMap *tm, uint32_t bar, int x, int y, int z,
                                                 int w)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(bar), "r"(x), "r"(y), "r"(z), "r"(w)
        : "memory");
}
__device__ __forceinline__ void tma_load_3d_pair(void *dst, const CUtensorMap *tm, uint32_t bar, int x, int y, int z)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(bar), "r"(x), "r"(y), "r"(z)
        : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t *slot_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot_smem)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8, %9, %10, %11, %12}, p;\n\t}" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u), "r"(0u), "r"(0u),
        "r"(0u), "r"(0u)
        : "memory");
}
// Arrive (once the MMAs issued so far complete) on `bar` in both CTAs of the pair.
__device__ __forceinline__ void mma_commit_pair(uint64_t *bar)
{
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"(static_cast<uint16_t>(3))
        : "memory");
}

// Bounded wait with cluster-scope acquire: these barriers are also arrived on from
// the other CTA (remote arrives, TMA completions, multicast commits).
__device__ __forceinline__ bool try_wait_cluster(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool wait2(uint64_t *bar, uint32_t parity, uint64_t limit_ns = kWaitLimitNs)
{
    if (try_wait_cluster(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 256; ++i)
            if (try_wait_cluster(bar, parity)) return true;
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
}

__device__ __forceinline__ void record2(int32_t *status, int code) { atomicCAS(status, 0, code); }
__device__ __forceinline__ float silu2(float a) { return a / (1.0f + __expf(-a)); }
__device__ __forceinline__ uint32_t pack_bf16_2(float a, float b)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Waits (at most limit_ns) until *ctr >= target, with acquire ordering at GPU scope.
__device__ __forceinline__ bool wait_count_at_least2(const int32_t *ctr, int target, uint64_t limit_ns)
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

// MODE 0: h = silu(x Wg^T) * (x Wu^T) -> bf16 rows of h; MODE 1: y rows of x Wd^T;
// MODE 3: the gate/up items, then the down items, in one launch (GemmArgs, mode 3).
template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS2, 1)
    grouped_gemm_2cta_kernel(const __grid_constant__ AMaps tmA, const __grid_constant__ CUtensorMap tmB0,
                             const __grid_constant__ CUtensorMap tmB1, const GemmArgs g, const int32_t *tiles2,
                             const int32_t *ntiles2, const __grid_constant__ SharedMaps sm,
                             const __grid_constant__ LayerMaps lm)
{
    constexpr int BNO0 = BN2 / 2, BNO1 = BN2;  // output columns of a gate/up item and of a down item
    extern __shared__ uint8_t smem2[];
    const uint32_t pad = (1024u - (smem_u32(smem2) & 1023u)) & 1023u;
    uint8_t *sA = smem2 + pad;
    uint8_t *sB = sA + ST2 * A2_BYTES;
    Ctrl2 *S = reinterpret_cast<Ctrl2 *>(sB + ST2 * B2_BYTES);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const uint32_t rank = cluster_rank();
    const int NP1 = MODE == 3 ? g.N2 : g.N, KP1 = MODE == 3 ? g.K2 : g.K;  // N and K of the down items
    const int nt0 = (g.N + BNO0 - 1) / BNO0, kb0 = (g.K + BKS2 - 1) / BKS2;
    const int nt1 = (NP1 + BNO1 - 1) / BNO1, kb1 = (KP1 + BKS2 - 1) / BKS2;
    // 64-column boxes of stage kb of a K range of Kd columns (a multiple of 64)
    auto boxes_of = [](int kb, int Kd) { return min(KW2, (Kd - kb * BKS2) / BK2); };

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < ST2; ++s) {
            mbar_init(&S->full[s], 2);
            mbar_init(&S->empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&S->accf[a], 1);
            mbar_init(&S->acce[a], 8);
        }
        for (int r = 0; r < RING2; ++r) {
            mbar_init(&S->itf[r], 1);
            mbar_init(&S->ite[r], 10);
        }
        mbar_init(&S->fin, 1);
        mbar_init(&S->bye, 1);
        fence_mbar_init();
        for (int b = 0; b < kABoxes; ++b) tma_prefetch_desc(&tmA.m[b]);
        tma_prefetch_desc(&tmB0);
        if (MODE != 1) tma_prefetch_desc(&tmB1);
        if (MODE == 3) tma_prefetch_desc(&lm.wd);
        if (g.sh_count) {
            tma_prefetch_desc(&sm.b0);
            if (MODE != 1) tma_prefetch_desc(&sm.b1);
        }
        if (MODE != 1 && g.a_rows) tma_prefetch_desc(&sm.xg);
    }
    if (warp == 1) tmem_alloc_pair(&S->tmem_base, TMEM_COLS2);
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers exist before any remote arrive
    tc_fence_after();
    const uint32_t tmem = S->tmem_base;
    // The prologue above overlapped the previous kernel; warp 0 waits for it inside the
    // producer, after the first stages' weight loads (only the A rows are the previous
    // kernel's output).
    if (warp != 0 || g.tiles_first) pdl_wait();
    pdl_trigger();
    if (g.trace && threadIdx.x == 0) g.trace[2 * blockIdx.x] = globaltimer_ns();

    // pair tiles: the list's, then the shared expert's; in mode 3 every gate/up item
    // precedes the down items
    const int nrouted = *ntiles2;
    const int sh_tps = g.sh_count ? (g.sh_T + 2 * HALF - 1) / (2 * HALF) : 1;
    const int mtiles = nrouted + g.sh_count * sh_tps;
    const int total0 = MODE == 3 ? mtiles * nt0 : 0;
    auto pos_of = [&](int item, int &mt, int &nt) {  // returns 1 for a down item
        const int p1 = MODE == 1 || (MODE == 3 && item >= total0);
        const int local = MODE == 3 && p1 ? item - total0 : item;
        const int ntl = p1 ? nt1 : nt0;
        mt = local / ntl;
        nt = local - mt * ntl;
        return p1;
    };

    if (warp == 0) {
        // -------------------------------- item hand-off (leader) + TMA producer (both)
        // Lane 0 hands items over and loads B (and A with row-block boxes); with direct
        // A rows (GemmArgs::a_rows) each lane gathers four A rows of this CTA's half of
        // a routed gate/up tile per stage, lane l rows 4l..4l+3.
        const bool gather = MODE != 1 && g.a_rows != nullptr;
        const int total = MODE == 3 ? total0 + mtiles * nt1 : mtiles * (MODE == 0 ? nt0 : nt1);
        int stage = 0, rs = 0, cursor = 0;
        uint32_t phase = 0, rphase = 0;
        bool ok = true;
        bool held = !g.tiles_first;  // A loads of the first item's first stages wait for the previous kernel
        for (;;) {
            int item = -1, okl = 1;
            if (lane == 0) {
                if (rank == 0) {
                    if (MODE != 3) {
                        item = claim_item(g.reverse, g.counter, total, MODE == 0 ? nt0 : nt1, tiles2, cursor, nrouted,
                                          g.sh_e0, sh_tps);
                    } else {  // the queue; descending within each phase in the reversed order
                        item = atomicAdd(g.counter, 1);
                        if (item >= total) item = -1;
                        else if (g.reverse == 1)
                            item = item < total0 ? total0 - 1 - item : total0 + (total - 1 - item);
                    }
                    if (wait2(&S->ite[rs], rphase ^ 1, g.wait_ns)) {
                        S->ring[rs] = item;
                        st_remote(peer_addr(&S->ring[rs], 1), item);
                        mbar_arrive(&S->itf[rs]);
                        arrive_remote(peer_addr(&S->itf[rs], 1));
                    } else {
                        okl = 0;
                    }
                } else {
                    if (wait2(&S->itf[rs], rphase, g.wait_ns)) {
                        item = S->ring[rs];
                        arrive_remote(peer_addr(&S->ite[rs], 0));
                    } else {
                        okl = 0;
                    }
                }
            }
            item = __shfl_sync(0xffffffffu, item, 0);
            if (!__shfl_sync(0xffffffffu, okl, 0)) { ok = false; break; }
            if (++rs == RING2) { rs = 0; rphase ^= 1; }
            if (item < 0) break;
            int mt, nt;
            const bool p1 = pos_of(item, mt, nt);
            const TileRef tr = tile_ref(tiles2, nrouted, mt, 2 * HALF, p1 ? 1 : 0, g.sh_T, g.sh_rows0, g.sh_e0);
            const int expert = tr.e;
            const int arow0 = tr.arow0 + (int)rank * HALF;  // this CTA's half of the pair tile
            const int rows = min(HALF, max(0, tr.rows - (int)rank * HALF));
            const int ab = a_box(rows);
            const CUtensorMap *amap = MODE == 3 && p1 ? &lm.h.m[ab] : (!p1 && tr.s >= 0) ? &sm.x.m[ab] : &tmA.m[ab];
            // direct rows: the x rows (tokens) of this lane's four rows, the tail's missing
            // rows repeating the half's last one (their products are masked)
            const bool g4 = gather && !p1 && tr.s < 0;
            const bool g4_lane = g4 && 4 * lane < rows;
            int tok[4] = {0, 0, 0, 0};
            auto load_tokens = [&]() {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int t = g.a_rows[arow0 + min(4 * lane + j, rows - 1)] / g.a_div;
                    tok[j] = (unsigned)t < (unsigned)g.a_tokens ? t : 0;
                }
            };
            if (g4_lane && !held) load_tokens();
            const uint32_t a_bytes = rows <= 0 ? 0u
                                   : g4        ? (uint32_t)((rows + 3) / 4) * 512u
                                               : (uint32_t)(a_box_rows(ab) * BK2 * 2);  // per 64-column box
            // B rows of this CTA: gate (CTA 0) or up (CTA 1) rows nt*128.. ; down: output columns
            const int nrow = !p1 ? nt * BNO0 : nt * BNO1 + (int)rank * 128;
            const CUtensorMap *bmap = !p1 ? (rank == 1 ? (tr.s >= 0 ? &sm.b1 : &tmB1) : (tr.s >= 0 ? &sm.b0 : &tmB0))
                                    : MODE == 3 ? (tr.s >= 0 ? &lm.wd_sh : &lm.wd)
                                                : (tr.s >= 0 ? &sm.b0 : &tmB0);
            const bool b_in = nrow < (p1 ? NP1 : g.N);  // a half entirely past N loads nothing (masked columns)
            const int num_kb = p1 ? kb1 : kb0;
            const int Kd = p1 ? KP1 : g.K;
            if (MODE == 3 && p1) {
                // the h rows of pair tile mt: wait until every gate/up item of mt published
                // them (4 epilogue warps in each of the 2 CTAs), then order those
                // generic-proxy writes before this CTA's TMA reads
                if (lane == 0) {
                    okl = wait_count_at_least2(g.ready + mt, 8 * nt0, g.wait_ns);
                    asm volatile("fence.proxy.async.global;" ::: "memory");
                }
                if (!__shfl_sync(0xffffffffu, okl, 0)) { ok = false; break; }
            }
            for (int kb = 0; kb < num_kb; ++kb) {
                const uint32_t fb = peer_addr(&S->full[stage], 0);
                const int nbx = boxes_of(kb, Kd);
                if (lane == 0) {
                    okl = wait2(&S->empty[stage], phase ^ 1, g.wait_ns);
                    if (okl) {
                        // the B box brings both chunks of its rows (one past the K range
                        // reads zeros and is not multiplied)
                        const uint32_t tx = a_bytes * (uint32_t)nbx + (b_in ? (uint32_t)B2_BYTES : 0u);
                        if (rank == 0)
                            mbar_arrive_expect_tx(&S->full[stage], tx);
                        else
                            arrive_expect_tx_remote(fb, tx);
                        for (int x = 0; x < nbx; ++x)
                            if (rows > 0 && !held && !g4)
                                tma_load_2d_pair(sA + stage * A2_BYTES + x * A2_SUB, amap, fb, kb * BKS2 + x * BK2,
                                                 arow0);
                        if (b_in) {  // [KW2][128 rows] of B in one box
                            uint8_t *b_dst = sB + stage * B2_BYTES;
                            const int z = kb * KW2;
                            if (tr.s < 0)
                                tma_load_4d_pair(b_dst, bmap, fb, 0, nrow, z, expert);
                            else if (!p1)  // shared slice s: rows s*I + nrow.. of the shared gate / up
                                tma_load_3d_pair(b_dst, bmap, fb, 0, tr.s * g.N + nrow, z);
                            else  // shared down: chunks of columns s*I..
                                tma_load_3d_pair(b_dst, bmap, fb, 0, nrow, tr.s * (KP1 / BK2) + z);
                        }
                    }
                }
                if (!__shfl_sync(0xffffffffu, okl, 0)) { ok = false; break; }
                if (g4_lane && !held)
                    for (int x = 0; x < nbx; ++x)
                        tma_gather4_pair(sA + stage * A2_BYTES + x * A2_SUB + lane * 512, &sm.xg, fb,
                                         kb * BKS2 + x * BK2, tok[0], tok[1], tok[2], tok[3]);
                if (++stage == ST2) { stage = 0; phase ^= 1; }
                if (held && kb + 1 == min(ST2, num_kb)) {  // first item: stage j holds K block j
                    pdl_wait();
                    held = false;
                    if (g4_lane) load_tokens();
                    for (int j = 0; j <= kb; ++j)
                        for (int x = 0; x < boxes_of(j, Kd); ++x) {
                            const int kx = j * BKS2 + x * BK2;
                            if (g4_lane)
                                tma_gather4_pair(sA + j * A2_BYTES + x * A2_SUB + lane * 512, &sm.xg,
                                                 peer_addr(&S->full[j], 0), kx, tok[0], tok[1], tok[2], tok[3]);
                            else if (!g4 && lane == 0 && rows > 0)
                                tma_load_2d_pair(sA + j * A2_BYTES + x * A2_SUB, amap, peer_addr(&S->full[j], 0), kx,
                                                 arow0);
                        }
                }
            }
            if (!ok) break;
        }
        if (!ok && lane == 0) record2(g.status, MOE_ERR_TIMEOUT);
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (leader only)
        if (lane == 0 && rank == 0) {
            constexpr uint32_t IDESC = idesc_bf16_f32(2 * HALF, BN2);
            int stage = 0, rs = 0, acc = 0;
            uint32_t phase = 0, rphase = 0, aphase = 0;
            bool ok = true;
            for (;;) {
                if (!wait2(&S->itf[rs], rphase, g.wait_ns)) { ok = false; break; }
                const int item = S->ring[rs];
                mbar_arrive(&S->ite[rs]);
                if (++rs == RING2) { rs = 0; rphase ^= 1; }
                if (item < 0) break;
                int mt_, nt_;
                const bool down = pos_of(item, mt_, nt_);
                const int num_kb = down ? kb1 : kb0, Kd = down ? KP1 : g.K;
                if (!wait2(&S->acce[acc], aphase ^ 1, g.wait_ns)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d = tmem + static_cast<uint32_t>(acc * BN2);
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!wait2(&S->full[stage], phase, g.wait_ns)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sA + stage * A2_BYTES);
                    const uint32_t b0 = smem_u32(sB + stage * B2_BYTES);
                    const int nbx = boxes_of(kb, Kd);
                    for (int x = 0; x < nbx; ++x)
#pragma unroll
                        for (int k = 0; k < BK2 / 16; ++k)
                            mma_bf16_pair(d, sw128_kmajor_desc(a0 + x * A2_SUB + k * 32),
                                          sw128_kmajor_desc(b0 + x * B2_SUB + k * 32), IDESC, (kb | x | k) != 0);
                    mma_commit_pair(&S->empty[stage]);
                    if (++stage == ST2) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                mma_commit_pair(&S->accf[acc]);
                if (++acc == 2) { acc = 0; aphase ^= 1; }
            }
            if (!ok) record2(g.status, MOE_ERR_TIMEOUT);
            mma_commit_pair(&S->fin);  // once every MMA issued here has completed
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue (both CTAs)
        const int q = warp & 3;
        const int row = q * 32 + lane;
        int rs = 0, acc = 0;
        uint32_t rphase = 0, aphase = 0;
        // y row of sorted row r: the row map's for the routed rows, r itself for the shared expert's
        auto flat_of = [&](int r) { return (g.sh_count == 0 || r < g.sh_rows0) ? g.row_map[r] : r; };
        for (;;) {
            if (!wait2(&S->itf[rs], rphase, g.wait_ns)) { record2(g.status, MOE_ERR_TIMEOUT); break; }
            const int item = S->ring[rs];
            __syncwarp();
            if (lane == 0) {
                if (rank == 0) mbar_arrive(&S->ite[rs]);
                else arrive_remote(peer_addr(&S->ite[rs], 0));
            }
            if (++rs == RING2) { rs = 0; rphase ^= 1; }
            if (item < 0) break;
            int mt, nt;
            const bool p1 = pos_of(item, mt, nt);
            const TileRef tr = tile_ref(tiles2, nrouted, mt, 2 * HALF, p1 ? 1 : 0, g.sh_T, g.sh_rows0, g.sh_e0);
            const int row0 = tr.row0 + (int)rank * HALF;
            const int rows = min(HALF, max(0, tr.rows - (int)rank * HALF));
            const bool row_ok = row < rows;
            if (!wait2(&S->accf[acc], aphase, g.wait_ns)) { record2(g.status, MOE_ERR_TIMEOUT); break; }
            tc_fence_after();
            const uint32_t tb = tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * BN2);
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
                            const float h0 = silu2(__uint_as_float(gr[2 * i])) * __uint_as_float(ur[2 * i]);
                            const float h1 = silu2(__uint_as_float(gr[2 * i + 1])) * __uint_as_float(ur[2 * i + 1]);
                            pk[i] = pack_bf16_2(h0, h1);
                        }
                        uint4 *dst = reinterpret_cast<uint4 *>(orow + col);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                    }
                }
            } else {
                __nv_bfloat16 *y = MODE == 3 ? g.out2 : g.out;
                const int flat = row_ok ? flat_of(row0 + row) : 0;
                __nv_bfloat16 *orow = y + (size_t)flat * NP1;
#pragma unroll 1
                for (int c = 0; c < BNO1 / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32_sync(tb + c * 32, r);
                    const int col = nt * BNO1 + c * 32;
                    if (row_ok && col < NP1) {
                        uint32_t pk[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            pk[i] = pack_bf16_2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
                        uint4 *dst = reinterpret_cast<uint4 *>(orow + col);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (rank == 0) mbar_arrive(&S->acce[acc]);
                else arrive_remote(peer_addr(&S->acce[acc], 0));
            }
            if (++acc == 2) { acc = 0; aphase ^= 1; }
            if (MODE == 3 && !p1) {
                // publish this warp's h rows of pair tile mt to the down items (release at
                // GPU scope after the proxy fence, counted once per warp)
                asm volatile("fence.proxy.async.global;" ::: "memory");
                __syncwarp();
                if (lane == 0) {
                    __threadfence();
                    atomicAdd(g.ready + mt, 1);
                }
            }
            if (p1 && g.comb_cnt)  // the accumulator is already released
                combine_arrive(MODE == 3 ? g.out2 : g.out, g.comb_gate, g.comb_out, g.comb_cnt, g.comb_k,
                               g.comb_target, NP1, nt1, nt, row_ok, row_ok ? flat_of(row0 + row) : 0, lane,
                               g.sh_count, g.sh_T, g.sh_rows0);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (g.trace && threadIdx.x == 0) g.trace[2 * blockIdx.x + 1] = globaltimer_ns();
    if (warp == 1) {
        // every MMA of the pair (which reads this CTA's shared memory and writes its
        // TMEM) has completed before TMEM is freed and the CTA may leave
        if (lane == 0 && !wait2(&S->fin, 0)) record2(g.status, MOE_ERR_TIMEOUT);
        __syncwarp();
        tc_fence_after();
        tmem_dealloc_pair(tmem, TMEM_COLS2);
    }
    __syncthreads();
    // leave only after the other CTA is done with this one (remote arrives, stores)
    if (threadIdx.x == 0) {
        arrive_remote(peer_addr(&S->bye, rank ^ 1u));
        if (!wait2(&S->bye, 0)) record2(g.status, MOE_ERR_TIMEOUT);
    }
    __syncthreads();
}

bool smem2_ready(int mode)
{
    static std::mutex mu;
    static uint64_t done[4] = {0, 0, 0, 0};  // per device
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    std::lock_guard<std::mutex> lk(mu);
    if (done[mode] >> dev & 1ull) return true;
    const int a = (int)SMEM2;
    cudaError_t e = mode == 0   ? cudaFuncSetAttribute(grouped_gemm_2cta_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, a)
                  : mode == 1 ? cudaFuncSetAttribute(grouped_gemm_2cta_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, a)
                              : cudaFuncSetAttribute(grouped_gemm_2cta_kernel<3>, cudaFuncAttributeMaxDynamicSharedMemorySize, a);
    if (e != cudaSuccess) return false;
    done[mode] |= 1ull << dev;
    return true;
}

}  // namespace

cudaError_t launch_grouped_gemm_2cta(const GemmArgs &g, const AMaps &tmA, const CUtensorMap &tmB0,
                                     const CUtensorMap &tmB1, const int32_t *tiles2, const int32_t *ntiles2,
                                     cudaStream_t st, const SharedMaps *sm, const LayerMaps *lm)
{
    int grid = (g.ctas > 0 ? g.ctas : num_sms()) / 2 * 2;
    if (grid < 2) grid = 2;
    if ((g.mode != 0 && g.mode != 1 && g.mode != 3) || g.reverse > 1) return cudaErrorInvalidValue;
    if (!smem2_ready(g.mode)) return cudaErrorInvalidValue;
    if (g.sh_count && !sm) return cudaErrorInvalidValue;
    if (g.mode == 3 && (!lm || !g.ready)) return cudaErrorInvalidValue;
    if (g.a_rows && (!sm || g.a_div <= 0 || g.a_tokens <= 0 || g.mode == 1)) return cudaErrorInvalidValue;
    static const SharedMaps none{};
    static const LayerMaps nolm{};
    const SharedMaps &s = sm ? *sm : none;
    const LayerMaps &l = lm ? *lm : nolm;
    if (g.mode == 0)
        return launch_pdl(grouped_gemm_2cta_kernel<0>, dim3(grid), dim3(THREADS2), SMEM2, st, tmA, tmB0, tmB1, g,
                          tiles2, ntiles2, s, l);
    if (g.mode == 1)
        return launch_pdl(grouped_gemm_2cta_kernel<1>, dim3(grid), dim3(THREADS2), SMEM2, st, tmA, tmB0, tmB1, g,
                          tiles2, ntiles2, s, l);
    return launch_pdl(grouped_gemm_2cta_kernel<3>, dim3(grid), dim3(THREADS2), SMEM2, st, tmA, tmB0, tmB1, g, tiles2,
                      ntiles2, s, l);
}

}  // namespace moe
