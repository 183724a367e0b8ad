// fp8_swapab.cu -- the fp8 gate/up GEMM with the MMA operands' roles swapped, for
// expert groups much shorter than a 128-row tile.
//
// The GC-MoE page (its compute-partition section) runs the expert GEMMs on
// Blackwell as operand-swapped tcgen05 block-scaled MMAs with SwiGLU and
// requantisation fused; this kernel is that idea for this layer's fp32 block scales.
// The one-CTA fp8 kernel (fp8.cu) puts a tile's token rows on the MMA's M side, so
// a group of 32 tokens still costs a 128-row MMA and a 128-row promotion of every K
// block.  Here the M side is 128 weight rows (output features of I) and the N side
// the tile's token rows rounded up to 16: D^T = W_gate . X^T and W_up . X^T, one
// accumulator each, so the tensor work and the TMEM traffic follow the group's
// size.  The arithmetic per output is the fp8 kernel's: for each 128-wide K block,
// P_kb = sum of e4m3 products in fp32 (TMEM), then acc += (s_a[row,kb] * s_w[kb]) *
// P_kb in fp32 registers; then h = silu(gate) * up and its e4m3 codes with one
// scale per token row per 128 features (the item's 128 features are exactly one
// scale group).
//
// A work item is (m-tile, 128 features, half of the m-tile): at most 64 token rows,
// so that the accumulators of a thread fit its registers (320 threads leave 168 a
// thread); the second half of a tile of up to 64 rows is an empty item that every
// role skips, and the two halves of a longer tile are consecutive items, so the
// second one finds the weights in L2.
//
// CTA roles (320 threads), as in the fp8 kernel: warp 0 claims items from the
// atomic queue and streams, per K block, the item's activation rows (16/32/64-row
// box) and 128 gate + 128 up weight rows with TMA (five stages); warp 1 owns TMEM
// and issues the MMAs (M = 128, N = rows rounded to 16, gate into columns 0-63 and
// up into 64-127 of one of four 128-column buffers); warps 2-9 promote, two warps
// per TMEM lane quarter (32 features), the pair splitting the token columns in
// 16-column chunks.  The per-token products
// s_a * s_w of 16 K blocks at a time are staged in shared memory by the epilogue
// warps themselves.  The per-token amax of h is reduced over each warp's 32
// features with redux.sync and over the four lane quarters through shared memory.
// Every wait is bounded.
#include <mutex>

#include "fp8_common.cuh"
#include "moe_internal.h"
#include "pdl.cuh"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

constexpr int XR = kTileRows / 2;       // token rows per item: the MMA's N at most
constexpr int FR = 128;                 // output features per item (gate and up each)
constexpr int KBYTES = 128;             // K bytes (e4m3 elements) per stage
constexpr int SST = 5;
constexpr int SRING = 4;
constexpr int NACC = 4;                 // TMEM accumulator buffers of 128 columns
constexpr int X_BYTES = XR * KBYTES;    // 8 KB
constexpr int W_BYTES = 2 * FR * KBYTES;  // 32 KB: 128 gate rows, then 128 up rows
constexpr int SEPI = 8;
constexpr int STHREADS = 64 + 32 * SEPI;
constexpr int SCH = 16;                 // K blocks per staged chunk of scale products
constexpr int SP = XR + 4;              // row pitch (floats) of a staged chunk
constexpr uint32_t STMEM_COLS = 512;

struct CtrlS {
    float sg[SCH * SP];    // [K block of the chunk][token row]: s_a * s_gate
    float su[SCH * SP];    // ... s_a * s_up
    float xam[2][XR][4];   // [item parity][token row][lane quarter]: amax of h over 32 features
    uint64_t full[SST], empty[SST];
    uint64_t accf[NACC], acce[NACC];
    uint64_t itf[SRING], ite[SRING];
    uint64_t sbar;         // the 8 epilogue warps, around each reload of the scale chunk
    uint64_t xbar[2];      // per half: its 4 warps posted their amax
    uint64_t fin, never;
    int32_t ring[SRING];
    uint32_t tmem_base;
};

// Item -> (expert, first row, rows, n-tile): item = (m-tile * n_tiles + n-tile) * 2 +
// half, the half taking rows [64 * half, 64 * half + 64) of the m-tile (rows <= 0:
// nothing there).
struct ItemS {
    int expert, row0, rows, nt;
};
__device__ __forceinline__ ItemS item_rows(const int32_t *tiles, int item, int n_tiles)
{
    const int hf = item & 1, mn = item >> 1;
    const int mt = mn / n_tiles;
    ItemS r;
    r.nt = mn - mt * n_tiles;
    r.expert = tiles[3 * mt];
    r.row0 = tiles[3 * mt + 1] + XR * hf;
    r.rows = min(XR, tiles[3 * mt + 2] - XR * hf);
    return r;
}

constexpr size_t SMEMS = 1024 + (size_t)SST * (X_BYTES + W_BYTES) + sizeof(CtrlS);
static_assert(SMEMS <= 227 * 1024, "shared memory of the swapped fp8 GEMM");
static_assert(sizeof(float) * SCH * SP % 16 == 0, "float4 alignment of the staged scales");

__global__ void __launch_bounds__(STHREADS, 1)
grouped_gemm_fp8_swapab_kernel(const __grid_constant__ AMaps tmX, const __grid_constant__ CUtensorMap tmWg,
                               const __grid_constant__ CUtensorMap tmWu, const Fp8GemmArgs g)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    uint8_t *sX = smem_raw + pad;
    uint8_t *sW = sX + SST * X_BYTES;
    CtrlS *S = reinterpret_cast<CtrlS *>(sW + SST * W_BYTES);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int n_tiles = g.N / FR;
    const int KB = g.K / KBYTES;
    const int NB = g.N / 128;

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < SST; ++s) {
            mbar_init(&S->full[s], 1);
            mbar_init(&S->empty[s], 1);
        }
        for (int a = 0; a < NACC; ++a) {
            mbar_init(&S->accf[a], 1);
            mbar_init(&S->acce[a], SEPI);
        }
        mbar_init(&S->xbar[0], 4);
        mbar_init(&S->xbar[1], 4);
        for (int r = 0; r < SRING; ++r) {
            mbar_init(&S->itf[r], 1);
            mbar_init(&S->ite[r], 1 + SEPI);
        }
        mbar_init(&S->sbar, SEPI);
        mbar_init(&S->fin, 1);
        mbar_init(&S->never, 1);
        fence_mbar_init();
        for (int b = 0; b < kABoxes; ++b) tma_prefetch_desc(&tmX.m[b]);
        tma_prefetch_desc(&tmWg);
        tma_prefetch_desc(&tmWu);
    }
    if (warp == 1) tmem_alloc(&S->tmem_base, STMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S->tmem_base;
    // The prologue above overlapped the previous kernel; warp 0 waits for it inside the
    // producer, after the first stages' weight loads (only the activation rows are the
    // previous kernel's output).
    if (warp != 0) pdl_wait();
    pdl_trigger();
    if (g.trace && threadIdx.x == 0) g.trace[2 * blockIdx.x] = globaltimer_ns();

    if (warp == 0) {
        // ------------------------------------------------ scheduler + TMA producer
        if (lane == 0) {
            const int total = *g.ntiles * n_tiles * 2;
            int stage = 0, rs = 0;
            uint32_t phase = 0, rphase = 0, armed = 0, armed_par = 0;
            bool ok = true;
            int cursor = (int)blockIdx.x * (g.reverse == 2);  // static modes
            bool held = true;  // activation loads of the first item's first stages wait for the previous kernel
            for (;;) {
                const int item = claim_item(g.reverse, g.counter, total, 2 * n_tiles, g.tiles, cursor);
                if (!mbar_wait(&S->ite[rs], rphase ^ 1, g.wait_ns)) { ok = false; break; }
                S->ring[rs] = item;
                mbar_arrive(&S->itf[rs]);
                if (++rs == SRING) { rs = 0; rphase ^= 1; }
                if (item < 0) break;
                const ItemS it = item_rows(g.tiles, item, n_tiles);
                if (it.rows <= 0) continue;  // the empty half of a short tile
                const int xb = a_box(it.rows);  // the activation box that covers the item's rows
                const int n0 = it.nt * FR;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&S->empty[stage], phase ^ 1, g.wait_ns)) { ok = false; break; }
                    mbar_arrive_expect_tx(&S->full[stage], a_box_rows(xb) * KBYTES + W_BYTES);
                    armed |= 1u << stage;
                    armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
                    uint8_t *w_dst = sW + stage * W_BYTES;
                    if (!held) tma_load_2d(sX + stage * X_BYTES, &tmX.m[xb], &S->full[stage], kb * KBYTES, it.row0);
                    tma_load_3d(w_dst, &tmWg, &S->full[stage], kb * KBYTES, n0, it.expert);
                    tma_load_3d(w_dst + W_BYTES / 2, &tmWu, &S->full[stage], kb * KBYTES, n0, it.expert);
                    if (++stage == SST) { stage = 0; phase ^= 1; }
                    if (held && kb + 1 == min(SST, KB)) {  // first item: stage j holds K block j
                        pdl_wait();
                        held = false;
                        for (int j = 0; j <= kb; ++j)
                            tma_load_2d(sX + j * X_BYTES, &tmX.m[xb], &S->full[j], j * KBYTES, it.row0);
                    }
                }
                if (!ok) break;
            }
            if (!ok) {
                record(g.status, MOE_ERR_TIMEOUT);
                if (mbar_wait(&S->ite[rs], rphase ^ 1)) {
                    S->ring[rs] = -1;
                    mbar_arrive(&S->itf[rs]);
                }
            }
            for (int s = 0; s < SST; ++s)
                if ((armed >> s) & 1u)
                    if (!mbar_wait(&S->full[s], (armed_par >> s) & 1u)) record(g.status, MOE_ERR_TIMEOUT);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            int stage = 0, rs = 0, acc = 0;
            uint32_t phase = 0, rphase = 0, aphase = 0;
            bool ok = !(g.stall_test && !mbar_wait(&S->never, 0, g.wait_ns));
            while (ok) {
                if (!mbar_wait(&S->itf[rs], rphase, g.wait_ns)) { ok = false; break; }
                const int item = S->ring[rs];
                mbar_arrive(&S->ite[rs]);
                if (++rs == SRING) { rs = 0; rphase ^= 1; }
                if (item < 0) break;
                const int rows = item_rows(g.tiles, item, n_tiles).rows;
                if (rows <= 0) continue;
                const uint32_t idesc = idesc_e4m3_f32(FR, (rows + 15) & ~15);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&S->acce[acc], aphase ^ 1, g.wait_ns)) { ok = false; break; }
                    tc_fence_after();
                    if (!mbar_wait(&S->full[stage], phase, g.wait_ns)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t d = tmem + static_cast<uint32_t>(acc * 2 * XR);
                    const uint32_t x0 = smem_u32(sX + stage * X_BYTES);
                    const uint32_t w0 = smem_u32(sW + stage * W_BYTES);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {  // 4 x K=32
                        const uint64_t xd = sw128_kmajor_desc(x0 + k * 32);
                        mma_e4m3(d, sw128_kmajor_desc(w0 + k * 32), xd, idesc, k != 0);
                        mma_e4m3(d + XR, sw128_kmajor_desc(w0 + W_BYTES / 2 + k * 32), xd, idesc, k != 0);
                    }
                    mma_commit(&S->empty[stage]);
                    mma_commit(&S->accf[acc]);
                    if (++stage == SST) { stage = 0; phase ^= 1; }
                    if (++acc == NACC) { acc = 0; aphase ^= 1; }
                }
            }
            if (!ok) record(g.status, MOE_ERR_TIMEOUT);
            mma_commit(&S->fin);
            if (!mbar_wait(&S->fin, 0)) record(g.status, MOE_ERR_TIMEOUT);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;            // TMEM lane quarter: features q*32 .. q*32+31
        const int half = (warp - 2) / 4;   // token chunks 2*ci + half
        const int et = threadIdx.x - 64;   // 0 .. 255 over the epilogue warps
        int rs = 0, acc = 0, parity = 0;
        uint32_t rphase = 0, aphase = 0, sphase = 0, xphase = 0;
        bool ok = true;
        auto epi_sync = [&]() {  // all 8 epilogue warps reached this point
            __syncwarp();
            if (lane == 0) mbar_arrive(&S->sbar);
            const bool r = mbar_wait(&S->sbar, sphase, g.wait_ns);
            sphase ^= 1;
            return r;
        };
        for (;;) {
            if (!mbar_wait(&S->itf[rs], rphase, g.wait_ns)) { ok = false; break; }
            const int item = S->ring[rs];
            __syncwarp();
            if (lane == 0) mbar_arrive(&S->ite[rs]);
            if (++rs == SRING) { rs = 0; rphase ^= 1; }
            if (item < 0) break;
            const ItemS it = item_rows(g.tiles, item, n_tiles);
            if (it.rows <= 0) continue;
            const int row0 = it.row0, rows = it.rows;
            const int np = (rows + 15) & ~15;  // the MMA's N
            const int n0 = it.nt * FR, nb = n0 / 128;
            const float *sa = g.sa + (size_t)row0 * KB;
            const float *sbg = g.sb0 + ((size_t)it.expert * NB + nb) * KB;
            const float *sbu = g.sb1 + ((size_t)it.expert * NB + nb) * KB;

            float ag[32], au[32];  // [chunk slot * 16 + column]: gate and up of this feature
#pragma unroll
            for (int i = 0; i < 32; ++i) ag[i] = au[i] = 0.0f;
            for (int kb = 0; kb < KB; ++kb) {
                const int kc = kb % SCH;
                if (kc == 0) {
                    // stage s_a * s_w of K blocks kb .. kb+15 for the tile's rows (rows past
                    // the tile get 0), once every warp is done with the previous chunk
                    if (!epi_sync()) { ok = false; break; }
                    const int nk = min(SCH, KB - kb);
                    for (int i = et; i < np * SCH; i += 32 * SEPI) {
                        const int t = i / SCH, c = i - t * SCH;
                        float vg = 0.0f, vu = 0.0f;
                        if (t < rows && c < nk) {
                            const float s = sa[(size_t)t * KB + kb + c];
                            vg = s * sbg[kb + c];
                            vu = s * sbu[kb + c];
                        }
                        S->sg[c * SP + t] = vg;
                        S->su[c * SP + t] = vu;
                    }
                    if (!epi_sync()) { ok = false; break; }
                }
                if (!mbar_wait(&S->accf[acc], aphase, g.wait_ns)) { ok = false; break; }
                tc_fence_after();
                const uint32_t tb = tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * 2 * XR);
#pragma unroll
                for (int ci = 0; ci < 2; ++ci) {
                    const int ch = 2 * ci + half;
                    if (ch * 16 >= np) continue;  // warp-uniform
                    uint32_t rg[16], ru[16];
                    tmem_ld16x2_sync(tb + ch * 16, tb + XR + ch * 16, rg, ru);
                    const float4 *pg = reinterpret_cast<const float4 *>(S->sg + kc * SP + ch * 16);
                    const float4 *pu = reinterpret_cast<const float4 *>(S->su + kc * SP + ch * 16);
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const float4 cg = pg[v], cu = pu[v];
                        const int i = ci * 16 + 4 * v;
                        ag[i] = fmaf(cg.x, __uint_as_float(rg[4 * v]), ag[i]);
                        ag[i + 1] = fmaf(cg.y, __uint_as_float(rg[4 * v + 1]), ag[i + 1]);
                        ag[i + 2] = fmaf(cg.z, __uint_as_float(rg[4 * v + 2]), ag[i + 2]);
                        ag[i + 3] = fmaf(cg.w, __uint_as_float(rg[4 * v + 3]), ag[i + 3]);
                        au[i] = fmaf(cu.x, __uint_as_float(ru[4 * v]), au[i]);
                        au[i + 1] = fmaf(cu.y, __uint_as_float(ru[4 * v + 1]), au[i + 1]);
                        au[i + 2] = fmaf(cu.z, __uint_as_float(ru[4 * v + 2]), au[i + 2]);
                        au[i + 3] = fmaf(cu.w, __uint_as_float(ru[4 * v + 3]), au[i + 3]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&S->acce[acc]);
                if (++acc == NACC) { acc = 0; aphase ^= 1; }
            }
            if (!ok) break;

            // h = silu(gate) * up; each token row's amax over this warp's 32 features
#pragma unroll
            for (int ci = 0; ci < 2; ++ci) {
                const int ch = 2 * ci + half;
                if (ch * 16 >= np) continue;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float h = silu(ag[ci * 16 + j]) * au[ci * 16 + j];
                    ag[ci * 16 + j] = h;
                    const uint32_t m = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(h)));
                    if (lane == j) S->xam[parity][ch * 16 + j][q] = __uint_as_float(m);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&S->xbar[half]);
            if (!mbar_wait(&S->xbar[half], xphase, g.wait_ns)) { ok = false; break; }
            xphase ^= 1;
            // the row's scale over all 128 features, then this feature's e4m3 code
            const int f = n0 + q * 32 + lane;
#pragma unroll
            for (int ci = 0; ci < 2; ++ci) {
                const int ch = 2 * ci + half;
                if (ch * 16 >= np) continue;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int t = ch * 16 + j;
                    if (t >= rows) continue;  // warp-uniform
                    const float4 a4 = *reinterpret_cast<const float4 *>(S->xam[parity][t]);
                    const float amax = fmaxf(fmaxf(a4.x, a4.y), fmaxf(a4.z, a4.w));
                    const float sc = amax == 0.0f ? 1.0f : __fdiv_rn(amax, 448.0f);
                    g.out_q[(size_t)(row0 + t) * g.N + f] = amax == 0.0f ? 0 : e4m3_one(qdiv(ag[ci * 16 + j], sc));
                    if (q == 0 && lane == j) g.out_s[(size_t)(row0 + t) * NB + nb] = sc;
                }
            }
            parity ^= 1;
        }
        if (!ok) record(g.status, MOE_ERR_TIMEOUT);
    }

    tc_fence_before();
    __syncthreads();
    if (g.trace && threadIdx.x == 0) g.trace[2 * blockIdx.x + 1] = globaltimer_ns();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, STMEM_COLS);
    }
}

bool swapab_smem_attr_ready()
{
    static std::mutex mu;
    static uint64_t done = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    std::lock_guard<std::mutex> lk(mu);
    if (done >> dev & 1ull) return true;
    if (cudaFuncSetAttribute(grouped_gemm_fp8_swapab_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SMEMS) != cudaSuccess)
        return false;
    done |= 1ull << dev;
    return true;
}

}  // namespace

cudaError_t launch_grouped_gemm_fp8_swapab(const Fp8GemmArgs &g, const AMaps &tmX, const CUtensorMap &tmWg,
                                           const CUtensorMap &tmWu, cudaStream_t st)
{
    if (g.mode != 0 || g.K % KBYTES || g.N % FR) return cudaErrorInvalidValue;
    if (!swapab_smem_attr_ready()) return cudaErrorInvalidValue;
    const int grid = g.ctas > 0 ? g.ctas : num_sms();
    return launch_pdl(grouped_gemm_fp8_swapab_kernel, dim3(grid), dim3(STHREADS), SMEMS, st, tmX, tmWg, tmWu, g);
}

}  // namespace moe
