// mx.cu -- the MX (microscaling) variant of the layer on sm_100a: e2m1 (FP4) expert
// weights and e4m3 activations, each with one power-of-two scale (an e8m0 code) per
// 32 values along K, multiplied on the tensor cores with the hardware's block
// scaling (tcgen05.mma kind::mxf8f6f4 with .block_scale).
//
// The GC-MoE page (its compute-partition section) runs the expert GEMMs on
// Blackwell as operand-swapped block-scaled tcgen05 MMAs over FP8/FP4 weights, with
// SwiGLU and the requantisation of h fused in.  The formats are those of the OCP
// Microscaling spec, which the MX kinds of the MMA take directly: the per-32 scales
// ride along in tensor memory and the MMA applies them, so each item accumulates
// its whole K range in one TMEM accumulator -- there is no per-K-block promotion as
// in the fp8 kernels, whose fp32 per-128 scales the hardware cannot take.
//
// Operands are swapped, as in fp8_swapab.cu: the MMA's M side is 128 weight rows
// (output features), its N side the item's token rows rounded up to 16, so the
// tensor work follows the expert group's size.  A work item is (m-tile, n-tile,
// half of the m-tile): at most 64 token rows against two 128-row weight tiles --
// gate and up rows n0.. in the gate/up GEMM (mode 0), output features n0.. and
// n0+128.. in the down GEMM (mode 1) -- each into its own accumulator.
//
// Data in shared memory: e4m3 token rows (128 bytes of K per stage) and e2m1 weight
// rows, which TMA expands on the way in from 16 packed codes in 8 bytes to 16 bytes
// (the 16U4_ALIGN16B type: the layout the MMA reads for 4-bit operands), both with
// the 128-byte swizzle.  The scales travel separately: every 4 stages TMA brings a
// [rows x 16 bytes] block of each operand's e8m0 codes (4 stages x 4 blocks of 32);
// four scale warps rearrange each stage's codes in shared memory into 32-row x
// 16-byte blocks (row r, word w: the codes of operand row 32w + r), and the MMA
// thread copies those into tensor memory with tcgen05.cp (32x128b, replicated to the
// four lane quarters), in order with the MMAs that read them.  In tensor memory the
// MMA finds the scale of M row m in lane m, column m / 32, and of N row n in lane
// n % 32, column n / 32; byte j of the 32-bit cell for the j-th K=32 MMA of the stage
// (its scale-factor id).
//
// CTA roles (320 threads): warp 0 claims items and streams tiles and scale blocks
// (TMA); warp 1 owns TMEM and issues the MMAs; warps 2-5 drain the accumulators --
// mode 0: h = silu(gate) * up, then per token and per 32 features (one warp's lanes)
// the MX e4m3 codes and scale of h; mode 1: bf16 rows of y -- and warps 6-9 are the
// scale warps, one per TMEM lane quarter.  Every wait is bounded.
#include <climits>
#include <mutex>

#include "fp8_common.cuh"
#include "moe_internal.h"
#include "pdl.cuh"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

constexpr int XR = kTileRows / 2;       // token rows per item: the MMA's N at most
constexpr int FR = 128;                 // weight rows per MMA: the MMA's M
constexpr int KE = 128;                 // K elements per stage (4 MMAs of K = 32)
constexpr int MST = 4;                  // stages, filled in pairs (K blocks 2j and 2j+1 on one barrier)
constexpr int MRING = 4;                // item ring
constexpr int SG = 4;                   // stages per scale block (16 bytes of e8m0 codes per row)
constexpr int X_BYTES = XR * KE;        // 8 KB: e4m3 token rows
constexpr int W_BYTES = FR * KE;        // 16 KB: one expanded e2m1 weight tile (128 rows x 128 B)
constexpr int W_TX = FR * KE / 2;       // 8 KB: its transaction bytes (TMA counts the packed codes it reads)
constexpr int SW_BYTES = FR * 16;       // 2 KB: scale block of one weight tile
constexpr int SX_BYTES = XR * 16;       // 1 KB: scale block of the token rows
constexpr int SBUF = 2 * SW_BYTES + SX_BYTES;
constexpr int CP_BYTES = 3 * 512;       // per stage: the tcgen05.cp sources of weight tiles 0, 1 and the tokens
constexpr int MTHREADS = 320;
constexpr uint32_t MTMEM_COLS = 512;
constexpr uint32_t ACC_COLS = 2 * XR;   // one accumulator buffer: two 64-column accumulators
constexpr uint32_t SF_COL0 = 256;       // scale slots: 16 columns per stage after two buffers
constexpr uint32_t SF_SLOT = 16;        // +0..3 weight tile 0, +4..7 weight tile 1, +8..9 token rows

struct CtrlM {
    uint64_t full[MST], empty[MST], sff[MST];
    uint64_t sgf[2], sge[2];
    uint64_t accf[2], acce[2];
    uint64_t itf[MRING], ite[MRING];
    uint64_t fin, never;
    int32_t ring[MRING];
    uint32_t tmem_base;
};

constexpr size_t SMEMM = 1024 + (size_t)MST * (X_BYTES + 2 * W_BYTES + CP_BYTES) + 2 * SBUF + sizeof(CtrlM);
static_assert(SMEMM <= 227 * 1024, "shared memory of the MX GEMM");
static_assert(SF_COL0 + MST * SF_SLOT <= MTMEM_COLS && 2 * ACC_COLS <= SF_COL0, "TMEM columns of the MX GEMM");

struct ItemM {
    int expert, row0, rows, nt;
};
__device__ __forceinline__ ItemM item_rows_m(const int32_t *tiles, int item, int n_tiles)
{
    const int hf = item & 1, mn = item >> 1;
    const int mt = mn / n_tiles;
    ItemM r;
    r.nt = mn - mt * n_tiles;
    r.expert = tiles[3 * mt];
    r.row0 = tiles[3 * mt + 1] + XR * hf;
    r.rows = min(XR, tiles[3 * mt + 2] - XR * hf);
    return r;
}

// kind::mxf8f6f4 instruction descriptor: A e2m1 (5), B e4m3 (0), both K-major, fp32
// accumulator, e8m0 scales (bit 23), M = 128, N; the scale-factor ids of A (bits
// 29-30) and B (bits 4-5) select the byte of each 32-bit scale cell.
__device__ __forceinline__ uint32_t idesc_mx(int N, uint32_t sf_id)
{
    return (5u << 7) | (0u << 10) | (static_cast<uint32_t>(N >> 3) << 17) | (1u << 23) |
           (static_cast<uint32_t>(FR >> 4) << 24) | (sf_id << 29) | (sf_id << 4);
}

__device__ __forceinline__ void mma_mx(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                                       uint32_t sfb, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}

// Shared-memory descriptor of a 32-row x 16-byte block without swizzle (8-row core
// matrices of 128 contiguous bytes), the source of a 32x128b tcgen05.cp.
__device__ __forceinline__ uint64_t cp_desc(uint32_t saddr)
{
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>(128u >> 4) << 16;  // leading byte offset
    d |= static_cast<uint64_t>(128u >> 4) << 32;  // stride byte offset: the next 8 rows
    d |= 1ull << 46;                              // descriptor version
    return d;
}

// Tensor memory columns taddr .. taddr+3 of all 128 lanes <- a 32-row x 16-byte block,
// row r to lanes r, r+32, r+64 and r+96.
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc)
{
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// The MX scale exponent of a block whose largest magnitude is amax: floor(log2 amax)
// minus the element format's largest exponent (8 for e4m3), within [-127, 127]; 0
// for an all-zero block.
__device__ __forceinline__ int mx_exponent(float amax)
{
    if (amax == 0.0f) return 0;
    const int x = ilogbf(amax) - 8;
    return x < -127 ? -127 : x > 127 ? 127 : x;
}

// e4m3 code of v / 2^X, rounded to nearest even and clamped to +-448; a value that
// rounds to zero is coded +0 whatever its sign (the MX element conversion here keeps
// no signed zero).
__device__ __forceinline__ uint8_t mx_e4m3(float v, int X)
{
    const uint8_t c = e4m3_one(fminf(fmaxf(ldexpf(v, -X), -448.0f), 448.0f));
    return (c & 0x7Fu) ? c : 0;
}

struct MxGemmArgs {
    int mode;          // 0: gate/up + SwiGLU + MX requantisation of h; 1: down -> y rows (bf16)
    int K, N;          // K of the GEMM; N = I (mode 0) or H (mode 1)
    const int32_t *tiles;
    const int32_t *ntiles;
    int32_t *counter;
    int32_t *status;
    uint8_t *out_q;    // mode 0: h codes [rows, N]
    uint8_t *out_x;    // mode 0: h scale codes [rows, N/32]
    __nv_bfloat16 *out;      // mode 1: y [T*k, N]
    const int32_t *row_map;  // mode 1: sorted row -> flat row
    int ctas;
    int reverse;
    uint64_t wait_ns;
    int stall_test;
    unsigned long long *trace;
};

// Tensor maps: tmX = the token rows' e4m3 codes (16/32/64-row boxes, 128 B of K);
// tmW0 / tmW1 = the two weight tiles' e2m1 codes (3-D, 128 rows x 128 codes);
// tmSX = the token rows' scale codes ([rows, K/32] bytes, 64 x 16 boxes); tmSW0 /
// tmSW1 = the weights' scale codes ([E, N, K/32], 128 x 16 boxes).
__global__ void __launch_bounds__(MTHREADS, 1)
grouped_gemm_mx_kernel(const __grid_constant__ AMaps tmX, const __grid_constant__ CUtensorMap tmW0,
                       const __grid_constant__ CUtensorMap tmW1, const __grid_constant__ CUtensorMap tmSX,
                       const __grid_constant__ CUtensorMap tmSW0, const __grid_constant__ CUtensorMap tmSW1,
                       const MxGemmArgs g)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    uint8_t *sX = smem_raw + pad;
    uint8_t *sW = sX + MST * X_BYTES;       // [stage pair][tile][2 stages][W_BYTES]
    uint8_t *sS = sW + MST * 2 * W_BYTES;   // [2][SBUF]: weight 0, weight 1, token scale blocks
    uint8_t *sC = sS + 2 * SBUF;            // [stage][CP_BYTES]: the stage's scales in the tcgen05.cp layout
    CtrlM *S = reinterpret_cast<CtrlM *>(sC + MST * CP_BYTES);
    // weight tile t of stage s: a pair of stages shares each tile's box (both K blocks of
    // its rows, 128 contiguous packed bytes a row)
    auto w_tile = [&](int s, int t) { return sW + (size_t)(s / 2) * 4 * W_BYTES + t * 2 * W_BYTES + (s & 1) * W_BYTES; };

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int mode = g.mode;
    const int fpi = mode == 0 ? FR : 2 * FR;  // output features per item
    const int n_tiles = (g.N + fpi - 1) / fpi;
    const int KB = g.K / KE;

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < MST; ++s) {
            mbar_init(&S->full[s], 1);
            mbar_init(&S->empty[s], 1);
            mbar_init(&S->sff[s], 4);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&S->sgf[b], 1);
            mbar_init(&S->sge[b], 4);
            mbar_init(&S->accf[b], 1);
            mbar_init(&S->acce[b], 4);
        }
        for (int r = 0; r < MRING; ++r) {
            mbar_init(&S->itf[r], 1);
            mbar_init(&S->ite[r], 9);  // the MMA thread, 4 epilogue warps, 4 scale warps
        }
        mbar_init(&S->fin, 1);
        mbar_init(&S->never, 1);
        fence_mbar_init();
        for (int b = 0; b < 3; ++b) tma_prefetch_desc(&tmX.m[b]);
        tma_prefetch_desc(&tmW0);
        tma_prefetch_desc(&tmW1);
        tma_prefetch_desc(&tmSX);
        tma_prefetch_desc(&tmSW0);
        tma_prefetch_desc(&tmSW1);
    }
    if (warp == 1) tmem_alloc(&S->tmem_base, MTMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S->tmem_base;
    pdl_wait();
    pdl_trigger();
    if (g.trace && threadIdx.x == 0) g.trace[2 * blockIdx.x] = globaltimer_ns();

    if (warp == 0) {
        // ------------------------------------------------ scheduler + TMA producer
        if (lane == 0) {
            const int total = *g.ntiles * n_tiles * 2;
            int stage = 0, rs = 0, gb = 0;
            uint32_t phase = 0, rphase = 0, gphase = 0, armed = 0, armed_par = 0, sarmed = 0, sarmed_par = 0;
            bool ok = true;
            int cursor = (int)blockIdx.x * (g.reverse == 2);
            for (;;) {
                const int item = claim_item(g.reverse, g.counter, total, 2 * n_tiles, g.tiles, cursor);
                if (!mbar_wait(&S->ite[rs], rphase ^ 1, g.wait_ns)) { ok = false; break; }
                S->ring[rs] = item;
                mbar_arrive(&S->itf[rs]);
                if (++rs == MRING) { rs = 0; rphase ^= 1; }
                if (item < 0) break;
                const ItemM it = item_rows_m(g.tiles, item, n_tiles);
                if (it.rows <= 0) continue;  // the empty half of a short tile
                const int xb = a_box(it.rows);
                const int n0 = it.nt * fpi, n1 = mode == 0 ? n0 : n0 + FR;
                for (int kb = 0; kb < KB; ++kb) {
                    if (kb % SG == 0) {  // the scale block of stages kb .. kb+3
                        if (!mbar_wait(&S->sge[gb], gphase ^ 1, g.wait_ns)) { ok = false; break; }
                        mbar_arrive_expect_tx(&S->sgf[gb], SBUF);
                        sarmed |= 1u << gb;
                        sarmed_par = (sarmed_par & ~(1u << gb)) | (gphase << gb);
                        uint8_t *sb = sS + gb * SBUF;
                        const int kx = kb * (KE / 32);  // first scale column (multiple of 16)
                        tma_load_3d(sb, &tmSW0, &S->sgf[gb], kx, n0, it.expert);
                        tma_load_3d(sb + SW_BYTES, &tmSW1, &S->sgf[gb], kx, n1, it.expert);
                        tma_load_2d(sb + 2 * SW_BYTES, &tmSX, &S->sgf[gb], kx, it.row0);
                        if (++gb == 2) { gb = 0; gphase ^= 1; }
                    }
                    if ((kb & 1) == 0) {
                        // K blocks kb and kb+1 (KB is a multiple of 4, and every item starts on
                        // an even stage) in stages stage and stage+1, on full[stage]
                        if (!mbar_wait(&S->empty[stage], phase ^ 1, g.wait_ns) ||
                            !mbar_wait(&S->empty[stage + 1], phase ^ 1, g.wait_ns)) { ok = false; break; }
                        mbar_arrive_expect_tx(&S->full[stage], 2 * (a_box_rows(xb) * KE + 2 * W_TX));
                        armed |= 1u << stage;
                        armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
                        tma_load_2d(sX + stage * X_BYTES, &tmX.m[xb], &S->full[stage], kb * KE, it.row0);
                        tma_load_2d(sX + (stage + 1) * X_BYTES, &tmX.m[xb], &S->full[stage], (kb + 1) * KE, it.row0);
                        tma_load_4d(w_tile(stage, 0), &tmW0, &S->full[stage], 0, n0, kb, it.expert);
                        tma_load_4d(w_tile(stage, 1), &tmW1, &S->full[stage], 0, n1, kb, it.expert);
                    }
                    if (++stage == MST) { stage = 0; phase ^= 1; }
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
            // never leave with TMA copies still landing in shared memory
            for (int s = 0; s < MST; ++s)
                if ((armed >> s) & 1u)
                    if (!mbar_wait(&S->full[s], (armed_par >> s) & 1u)) record(g.status, MOE_ERR_TIMEOUT);
            for (int b = 0; b < 2; ++b)
                if ((sarmed >> b) & 1u)
                    if (!mbar_wait(&S->sgf[b], (sarmed_par >> b) & 1u)) record(g.status, MOE_ERR_TIMEOUT);
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
                if (++rs == MRING) { rs = 0; rphase ^= 1; }
                if (item < 0) break;
                const int rows = item_rows_m(g.tiles, item, n_tiles).rows;
                if (rows <= 0) continue;
                const int np = (rows + 15) & ~15;
                if (!mbar_wait(&S->acce[acc], aphase ^ 1, g.wait_ns)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d0 = tmem + static_cast<uint32_t>(acc) * ACC_COLS, d1 = d0 + XR;
                for (int kb = 0; kb < KB; ++kb) {
                    // the pair's data lands on the even stage's barrier
                    if ((kb & 1) == 0 && !mbar_wait(&S->full[stage], phase, g.wait_ns)) { ok = false; break; }
                    if (!mbar_wait(&S->sff[stage], phase, g.wait_ns)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t x0 = smem_u32(sX + stage * X_BYTES);
                    const uint32_t w0 = smem_u32(w_tile(stage, 0)), w1 = smem_u32(w_tile(stage, 1));
                    const uint32_t sf = tmem + SF_COL0 + static_cast<uint32_t>(stage) * SF_SLOT;
                    const uint32_t cp0 = smem_u32(sC + stage * CP_BYTES);
                    tmem_cp_32x128b_x4(sf, cp_desc(cp0));             // weight tile 0
                    tmem_cp_32x128b_x4(sf + 4, cp_desc(cp0 + 512));   // weight tile 1
                    tmem_cp_32x128b_x4(sf + 8, cp_desc(cp0 + 1024));  // token rows
#pragma unroll
                    for (int k = 0; k < KE / 32; ++k) {
                        const uint64_t xd = sw128_kmajor_desc(x0 + k * 32);
                        const uint32_t idesc = idesc_mx(np, static_cast<uint32_t>(k));
                        const uint32_t accum = (kb | k) != 0;
                        mma_mx(d0, sw128_kmajor_desc(w0 + k * 32), xd, idesc, sf, sf + 8, accum);
                        mma_mx(d1, sw128_kmajor_desc(w1 + k * 32), xd, idesc, sf + 4, sf + 8, accum);
                    }
                    mma_commit(&S->empty[stage]);
                    if (++stage == MST) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                mma_commit(&S->accf[acc]);
                if (++acc == 2) { acc = 0; aphase ^= 1; }
            }
            if (!ok) record(g.status, MOE_ERR_TIMEOUT);
            mma_commit(&S->fin);
            if (!mbar_wait(&S->fin, 0)) record(g.status, MOE_ERR_TIMEOUT);
        }
        __syncwarp();
    } else if (warp < 6) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;  // TMEM lane quarter: weight rows (features) q*32 .. q*32+31
        int rs = 0, acc = 0;
        uint32_t rphase = 0, aphase = 0;
        bool ok = true;
        for (;;) {
            if (!mbar_wait(&S->itf[rs], rphase, g.wait_ns)) { ok = false; break; }
            const int item = S->ring[rs];
            __syncwarp();
            if (lane == 0) mbar_arrive(&S->ite[rs]);
            if (++rs == MRING) { rs = 0; rphase ^= 1; }
            if (item < 0) break;
            const ItemM it = item_rows_m(g.tiles, item, n_tiles);
            if (it.rows <= 0) continue;
            const int np = (it.rows + 15) & ~15;
            const int n0 = it.nt * fpi;
            if (!mbar_wait(&S->accf[acc], aphase, g.wait_ns)) { ok = false; break; }
            tc_fence_after();
            const uint32_t tb = tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc) * ACC_COLS;
            for (int c = 0; c < np; c += 16) {  // 16 token columns at a time
                uint32_t r0[16], r1[16];
                tmem_ld16x2_sync(tb + c, tb + XR + c, r0, r1);
                if (mode == 0) {
                    // h of feature f = n0 + 32q + lane for 16 tokens; per token, the MX block
                    // is this warp's 32 features
                    const int f = n0 + q * 32 + lane;
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int t = c + j;
                        const float h = silu(__uint_as_float(r0[j])) * __uint_as_float(r1[j]);
                        const float amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(h))));
                        if (t >= it.rows) continue;  // warp-uniform
                        const int X = mx_exponent(amax);
                        const size_t row = (size_t)(it.row0 + t);
                        g.out_q[row * g.N + f] = amax == 0.0f ? 0 : mx_e4m3(h, X);
                        if (lane == 0) g.out_x[row * (g.N / 32) + (n0 + q * 32) / 32] = static_cast<uint8_t>(X + 127);
                    }
                } else {
                    const int f0 = n0 + q * 32 + lane, f1 = f0 + FR;
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int t = c + j;
                        if (t >= it.rows) continue;  // warp-uniform
                        __nv_bfloat16 *yrow = g.out + (size_t)g.row_map[it.row0 + t] * g.N;
                        if (f0 < g.N) yrow[f0] = __float2bfloat16_rn(__uint_as_float(r0[j]));
                        if (f1 < g.N) yrow[f1] = __float2bfloat16_rn(__uint_as_float(r1[j]));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S->acce[acc]);
            if (++acc == 2) { acc = 0; aphase ^= 1; }
        }
        if (!ok) record(g.status, MOE_ERR_TIMEOUT);
    } else {
        // ---------------------------------------------------------- scale warps
        // Per stage, thread (q, lane) moves the codes of weight row 32q + lane of each
        // tile to word q of row `lane` of that tile's 32 x 16-byte block; the quarter-0
        // warp also moves tokens lane and lane + 32 to words 0 and 1 of the token block.
        const int q = warp & 3;
        int rs = 0, stage = 0, gb = 0;
        uint32_t rphase = 0, phase = 0, gphase = 0;
        bool ok = true;
        for (;;) {
            if (!mbar_wait(&S->itf[rs], rphase, g.wait_ns)) { ok = false; break; }
            const int item = S->ring[rs];
            __syncwarp();
            if (lane == 0) mbar_arrive(&S->ite[rs]);
            if (++rs == MRING) { rs = 0; rphase ^= 1; }
            if (item < 0) break;
            if (item_rows_m(g.tiles, item, n_tiles).rows <= 0) continue;
            for (int kb = 0; kb < KB && ok; ++kb) {
                if (kb % SG == 0 && !mbar_wait(&S->sgf[gb], gphase, g.wait_ns)) { ok = false; break; }
                // the MMAs (and copies) of this stage's previous use are done with its buffer
                if (!mbar_wait(&S->empty[stage], phase ^ 1, g.wait_ns)) { ok = false; break; }
                const uint8_t *sb = sS + gb * SBUF;
                uint8_t *cp = sC + stage * CP_BYTES;
                const int u = kb % SG;
                const int m = q * 32 + lane;
                *reinterpret_cast<uint32_t *>(cp + lane * 16 + q * 4) =
                    *reinterpret_cast<const uint32_t *>(sb + m * 16 + u * 4);
                *reinterpret_cast<uint32_t *>(cp + 512 + lane * 16 + q * 4) =
                    *reinterpret_cast<const uint32_t *>(sb + SW_BYTES + m * 16 + u * 4);
                if (q == 0) {
                    const uint8_t *sx = sb + 2 * SW_BYTES;
                    uint4 t;
                    t.x = *reinterpret_cast<const uint32_t *>(sx + lane * 16 + u * 4);
                    t.y = *reinterpret_cast<const uint32_t *>(sx + (lane + 32) * 16 + u * 4);
                    t.z = t.w = 0x7F7F7F7Fu;  // unused columns (N <= 64)
                    *reinterpret_cast<uint4 *>(cp + 1024 + lane * 16) = t;
                }
                fence_proxy_async_smem();  // the writes above, before the tensor cores' copy reads them
                __syncwarp();
                if (lane == 0) mbar_arrive(&S->sff[stage]);
                if (u == SG - 1 || kb == KB - 1) {  // done with this scale block
                    if (lane == 0) mbar_arrive(&S->sge[gb]);
                    if (++gb == 2) { gb = 0; gphase ^= 1; }
                }
                if (++stage == MST) { stage = 0; phase ^= 1; }
            }
            if (!ok) break;
        }
        if (!ok) record(g.status, MOE_ERR_TIMEOUT);
    }

    tc_fence_before();
    __syncthreads();
    if (g.trace && threadIdx.x == 0) g.trace[2 * blockIdx.x + 1] = globaltimer_ns();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, MTMEM_COLS);
    }
}

// MX e4m3 quantisation of bf16 rows: a thread per block of 32 values.
__global__ void __launch_bounds__(256) quantize_rows_mx_kernel(const __nv_bfloat16 *__restrict__ src, int R, int K,
                                                               uint8_t *__restrict__ q, uint8_t *__restrict__ x)
{
    pdl_wait();
    pdl_trigger();
    const long nblk = (long)R * (K / 32);
    const long b = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= nblk) return;
    const uint4 *p = reinterpret_cast<const uint4 *>(src + b * 32);
    float v[32];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint4 w = p[i];
        const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            v[8 * i + 2 * j] = __uint_as_float(u[j] << 16);
            v[8 * i + 2 * j + 1] = __uint_as_float(u[j] & 0xFFFF0000u);
        }
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
    const int X = mx_exponent(amax);
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        uint32_t c = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j)
            c |= static_cast<uint32_t>(amax == 0.0f ? 0 : mx_e4m3(v[4 * i + j], X)) << (8 * j);
        w[i] = c;
    }
    uint4 *dq = reinterpret_cast<uint4 *>(q + b * 32);
    dq[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dq[1] = make_uint4(w[4], w[5], w[6], w[7]);
    x[b] = static_cast<uint8_t>(X + 127);
}

// MX rows into expert order, a warp per sorted row r: xs[r] = xq[s2f[r] / k] (K codes)
// and xs_x[r] = xq_x[...] (K/32 scale codes).
__global__ void gather_rows_mx_kernel(const uint8_t *__restrict__ xq, const uint8_t *__restrict__ xq_x,
                                      const int32_t *__restrict__ s2f, int A, int K, int k, uint8_t *__restrict__ xs,
                                      uint8_t *__restrict__ xs_x)
{
    pdl_wait();
    pdl_trigger();
    const int r = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (r >= A) return;
    const int f = s2f[r];
    if ((unsigned)f >= (unsigned)A) return;
    const int t = f / k;
    const uint4 *src = reinterpret_cast<const uint4 *>(xq + (size_t)t * K);
    uint4 *dst = reinterpret_cast<uint4 *>(xs + (size_t)r * K);
    for (int c = lane; c < K / 16; c += 32) dst[c] = src[c];
    const uint4 *ssrc = reinterpret_cast<const uint4 *>(xq_x + (size_t)t * (K / 32));
    uint4 *sdst = reinterpret_cast<uint4 *>(xs_x + (size_t)r * (K / 32));
    for (int c = lane; c < K / 512; c += 32) sdst[c] = ssrc[c];
}

bool mx_smem_attr_ready()
{
    static std::mutex mu;
    static uint64_t done = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    std::lock_guard<std::mutex> lk(mu);
    if (done >> dev & 1ull) return true;
    if (cudaFuncSetAttribute(grouped_gemm_mx_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEMM) !=
        cudaSuccess)
        return false;
    done |= 1ull << dev;
    return true;
}

}  // namespace

cudaError_t launch_quantize_rows_mx(const __nv_bfloat16 *src, int R, int K, uint8_t *q, uint8_t *x, cudaStream_t st)
{
    const long nblk = (long)R * (K / 32);
    return launch_pdl(quantize_rows_mx_kernel, dim3((unsigned)((nblk + 255) / 256)), dim3(256), 0, st, src, R, K, q,
                      x);
}

cudaError_t launch_gather_rows_mx(const uint8_t *xq, const uint8_t *xq_x, const int32_t *s2f, int A, int K, int k,
                                  uint8_t *xs, uint8_t *xs_x, cudaStream_t st)
{
    const int rows_per_block = 8;
    return launch_pdl(gather_rows_mx_kernel, dim3((A + rows_per_block - 1) / rows_per_block),
                      dim3(rows_per_block * 32), 0, st, xq, xq_x, s2f, A, K, k, xs, xs_x);
}

cudaError_t launch_grouped_gemm_mx(const MxLaunch &l, cudaStream_t st)
{
    if (l.K % 512 || l.N % 128 || (l.mode != 0 && l.mode != 1)) return cudaErrorInvalidValue;
    if (!mx_smem_attr_ready()) return cudaErrorInvalidValue;
    MxGemmArgs g{l.mode, l.K, l.N, l.tiles, l.ntiles, l.counter, l.status, l.out_q, l.out_x, l.out, l.row_map,
                 l.ctas, l.reverse, l.wait_ns, l.stall_test, l.trace};
    const int grid = l.ctas > 0 ? l.ctas : num_sms();
    return launch_pdl(grouped_gemm_mx_kernel, dim3(grid), dim3(MTHREADS), SMEMM, st, l.tmX, l.tmW0, l.tmW1, l.tmSX,
                      l.tmSW0, l.tmSW1, g);
}

}  // namespace moe
