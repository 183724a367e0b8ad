// fp8.cu -- the FP8 block-scaled variant of the layer on sm_100a.
//
// Weights arrive as e4m3 codes with one fp32 scale per 128x128 block;
// activations are quantised per row per 128 columns (x before the gate/up GEMM,
// h after SwiGLU) with s = amax/448 and q = e4m3_rn(clamp(v/s, +-448)).  The
// GC-MoE page describes this family of kernels on Blackwell: block-scaled tcgen05
// MMA with SwiGLU and requantisation fused into the GEMM; the vLLM page
// (section 03) lists fp8 configs with [128,128] weight blocks.
//
// Hardware block scaling (kind::mxf8f6f4) takes one power-of-two scale per 32
// elements, which cannot hold these fp32 per-128 scales.  So each 128-wide K
// block is one MMA group of kind::f8f6f4 (4 x K=32) into a fresh TMEM buffer,
// and the epilogue warps promote it: acc += (s_a[row,kb] * s_b[nblk,kb]) * P_kb,
// in fp32 registers, while the tensor cores fill the other TMEM buffer.
//
// CTA roles (320 threads): warp 0 claims work items and streams 128x128-byte A
// tiles and 256x128-byte B tiles with TMA (one stage = one K block); warp 1 owns
// TMEM and issues the MMAs; warps 2-9 are the epilogue, two warps per TMEM lane
// quarter, each owning 128 of the 256 accumulator columns of its rows.
// Mode 0 (gate/up): columns 0-127 are gate, 128-255 up, of the same 128 rows of
// I; a thread owns 64 gate + 64 up columns, forms h = silu(g) * u, and the two
// warps sharing a row exchange their partial amax through shared memory to
// quantise the 128-column group.  Mode 1 (down): y rows in bf16.  Mode 2 (bf16
// operands, no scales, plain 128-row blocks, K optionally split over items):
// the router's tensor-core logits, each 64-wide K block summed out of TMEM in
// fp32 so the accumulation error does not grow with H.
// Every wait is bounded, as in the bf16 kernel.
#include <cuda_fp8.h>

#include <mutex>

#include "combine.cuh"
#include "fp8_common.cuh"
#include "moe_internal.h"
#include "pdl.cuh"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

constexpr int BM = kTileRows;
constexpr int BKB = 128;                // bytes (= e4m3 elements) of K per stage
constexpr int BN = 256;
constexpr int STAGES = 4;
constexpr int RING = 4;
constexpr int A_BYTES = BM * BKB;       // 16 KB
constexpr int B_BYTES = BN * BKB;       // 32 KB
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr uint32_t TMEM_COLS = 512;

// Tensor-map store of a box from shared memory (bulk-group completion): the box's
// elements outside the tensor's extent are not written.  Generic-proxy writes to the
// box must be made visible to the TMA first (fence_proxy_async_shared_cta).
__device__ __forceinline__ void tma_store_3d(const CUtensorMap *tm, const void *src, int x, int y, int z)
{
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(tm)),
                 "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Waits until this thread's committed bulk groups have completed (their writes done).
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_shared_cta()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

struct Ctrl8 {
    uint64_t full[STAGES], empty[STAGES];
    uint64_t accf[2], acce[2];
    uint64_t itf[RING], ite[RING];
    uint64_t xbar[4];  // per lane quarter: the two epilogue warps of those rows
    uint64_t fin, never;
    int32_t ring[RING];
    uint32_t tmem_base;
    float xam[2][2][BM];  // [item parity][half][row]: partial amax of h
};

constexpr size_t SMEM8 = 1024 + (size_t)STAGES * (A_BYTES + B_BYTES) + sizeof(Ctrl8);
// Mode 2 adds a transpose buffer per epilogue warp: 32 rows x 16 fp32 logits, rows
// padded to 80 bytes (five 16-byte slots, so that eight consecutive rows' slots fall
// in distinct bank groups).
constexpr int EPI2_ROW = 20;  // floats per buffered row
constexpr size_t EPI2_BYTES = (size_t)EPI_WARPS * 32 * EPI2_ROW * 4;
constexpr size_t EPI2_OFF = (sizeof(Ctrl8) + 15) / 16 * 16;  // after the control block, 16-byte aligned
constexpr size_t smem8_bytes(int mode) { return SMEM8 + (mode == 2 ? 16 + EPI2_BYTES : 0); }
static_assert(smem8_bytes(2) <= 232448, "mode 2 shared memory");

// ------------------------------------------------------------ quantiser

// The fp8 activations of the forward: x is quantised once per token, then row r of
// the expert-sorted copy takes token s2f[r] / k's codes and scales (a warp per row).
__global__ void gather_rows_fp8_kernel(const uint8_t *__restrict__ xq, const float *__restrict__ xq_s,
                                       const int32_t *__restrict__ s2f, int A, int K, int k, uint8_t *__restrict__ xs,
                                       float *__restrict__ xs_s)
{
    pdl_wait();
    pdl_trigger();
    const int row = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (row >= A) return;
    const int t = s2f[row] / k;
    const uint4 *src = reinterpret_cast<const uint4 *>(xq + (size_t)t * K);
    uint4 *dst = reinterpret_cast<uint4 *>(xs + (size_t)row * K);
    for (int c = lane; c < K / 16; c += 32) dst[c] = src[c];
    for (int c = lane; c < K / 128; c += 32) xs_s[(size_t)row * (K / 128) + c] = xq_s[(size_t)t * (K / 128) + c];
}

// Rows of a bf16 matrix quantised per 128-column group.  Row r reads source row
// map ? map[r] / k : r.  A warp takes eight groups (1024 columns) of one row: four
// lanes per group, 32 values each in four 16-byte loads, the group's amax over the
// four lanes, then 32 codes in two 16-byte stores.
__global__ void quantize_rows_kernel(const __nv_bfloat16 *__restrict__ src, const int32_t *__restrict__ map,
                                     int k, int R, int K, uint8_t *__restrict__ q, float *__restrict__ s)
{
    pdl_wait();
    pdl_trigger();
    const int warps_per_row = (K / 128 + 7) / 8;
    const long wid = (long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (wid >= (long)R * warps_per_row) return;
    const int row = (int)(wid / warps_per_row);
    const int g = (int)(wid % warps_per_row) * 8 + lane / 4;  // this lane's group
    const int sub = lane % 4;
    const bool has = g < K / 128;                              // warp-uniform per group of 4 lanes
    const int sr = map ? map[row] / k : row;
    float v[32];
    float m = 0.0f;
    if (has) {
        const uint4 *a = reinterpret_cast<const uint4 *>(src + (size_t)sr * K + g * 128 + sub * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 raw = a[i];
            const __nv_bfloat162 *p = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 f = __bfloat1622float2(p[j]);
                v[8 * i + 2 * j] = f.x;
                v[8 * i + 2 * j + 1] = f.y;
                m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
            }
        }
    }
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
    if (!has) return;
    float sc = 1.0f;
    uint32_t w[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    if (m != 0.0f) {
        sc = __fdiv_rn(m, 448.0f);
#pragma unroll
        for (int i = 0; i < 8; ++i)
            w[i] = e4m3_pair(qdiv(v[4 * i], sc), qdiv(v[4 * i + 1], sc)) |
                   (e4m3_pair(qdiv(v[4 * i + 2], sc), qdiv(v[4 * i + 3], sc)) << 16);
    }
    uint4 *dst = reinterpret_cast<uint4 *>(q + (size_t)row * K + g * 128 + sub * 32);
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    if (sub == 0) s[(size_t)row * (K / 128) + g] = sc;
}

// ----------------------------------------------------------- grouped GEMM

template <int MODE, bool BF16, bool COMB = false>
__global__ void __launch_bounds__(THREADS, 1)
grouped_gemm_fp8_kernel(const __grid_constant__ AMaps tmA, const __grid_constant__ CUtensorMap tmB0,
                        const __grid_constant__ CUtensorMap tmB1, const Fp8GemmArgs g)
{
    constexpr int BNO = MODE == 0 ? BN / 2 : BN;  // output columns per tile
    constexpr int KEL = BF16 ? 64 : 128;          // elements of K per stage (128 bytes)
    const bool dense = g.tiles == nullptr;        // mode 2: plain 128-row blocks of A
    const int ksplit = g.ksplit > 0 ? g.ksplit : 1;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    uint8_t *sA = smem_raw + pad;
    uint8_t *sB = sA + STAGES * A_BYTES;
    Ctrl8 *S = reinterpret_cast<Ctrl8 *>(sB + STAGES * B_BYTES);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int n_tiles = (g.N + BNO - 1) / BNO;
    const int KB = g.K / KEL;
    const int KBS = (KB + ksplit - 1) / ksplit;  // K blocks per item
    const int NB = g.N / 128;  // 128-row weight blocks along N

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&S->full[s], 1);
            mbar_init(&S->empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&S->accf[a], 1);
            mbar_init(&S->acce[a], EPI_WARPS);
        }
        for (int r = 0; r < RING; ++r) {
            mbar_init(&S->itf[r], 1);
            mbar_init(&S->ite[r], 1 + EPI_WARPS);
        }
        for (int q = 0; q < 4; ++q) mbar_init(&S->xbar[q], 2);
        mbar_init(&S->fin, 1);
        mbar_init(&S->never, 1);
        fence_mbar_init();
        for (int b = 0; b < kABoxes; ++b) tma_prefetch_desc(&tmA.m[b]);
        tma_prefetch_desc(&tmB0);
        if (MODE == 0) tma_prefetch_desc(&tmB1);
    }
    if (warp == 1) tmem_alloc(&S->tmem_base, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S->tmem_base;
    // The prologue above overlapped the previous kernel.  Warp 0 waits for it inside
    // the producer, after the loads of the first stages that do not depend on it: the
    // weights in modes 0 and 1 (A is the previous kernel's output), x in mode 2 (B, the
    // transposed router matrix, is the previous kernel's output).
    constexpr bool kEarlyB = MODE != 2;
    if (warp != 0) pdl_wait();
    pdl_trigger();
    if (g.trace && threadIdx.x == 0) g.trace[2 * blockIdx.x] = globaltimer_ns();

    if (warp == 0) {
        // ------------------------------------------------ scheduler + TMA producer
        if (lane == 0) {
            const int total = (dense ? (g.M + BM - 1) / BM : *g.ntiles) * n_tiles * ksplit;
            int stage = 0, rs = 0;
            uint32_t phase = 0, rphase = 0, armed = 0, armed_par = 0;
            bool ok = true;
            int cursor = (int)blockIdx.x * (g.reverse == 2);  // static modes
            bool held = true;  // the first item's first stages: dependent loads wait for the previous kernel
            for (;;) {
                const int item = claim_item(g.reverse, g.counter, total, n_tiles * ksplit, dense ? nullptr : g.tiles, cursor);
                if (!mbar_wait(&S->ite[rs], rphase ^ 1, g.wait_ns)) { ok = false; break; }
                S->ring[rs] = item;
                mbar_arrive(&S->itf[rs]);
                if (++rs == RING) { rs = 0; rphase ^= 1; }
                if (item < 0) break;
                const int ks = item % ksplit, mn = item / ksplit;
                const int mt = mn / n_tiles, nt = mn - mt * n_tiles;
                const int expert = dense ? 0 : g.tiles[3 * mt], row0 = dense ? mt * BM : g.tiles[3 * mt + 1];
                const int rows = dense ? min(BM, g.M - row0) : g.tiles[3 * mt + 2];
                const int ab = a_box(rows);  // the A box that covers the tile's rows
                const int n0 = nt * BNO;
                const int kb0 = ks * KBS, kb1 = min(KB, kb0 + KBS);
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait(&S->empty[stage], phase ^ 1, g.wait_ns)) { ok = false; break; }
                    mbar_arrive_expect_tx(&S->full[stage], a_box_rows(ab) * 128 + B_BYTES);
                    armed |= 1u << stage;
                    armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
                    uint8_t *b_dst = sB + stage * B_BYTES;
                    if (!held || !kEarlyB) tma_load_2d(sA + stage * A_BYTES, &tmA.m[ab], &S->full[stage], kb * KEL, row0);
                    if (!held || kEarlyB) {
                        tma_load_3d(b_dst, &tmB0, &S->full[stage], kb * KEL, n0, expert);
                        if (MODE == 0) tma_load_3d(b_dst + B_BYTES / 2, &tmB1, &S->full[stage], kb * KEL, n0, expert);
                    }
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                    if (held && kb + 1 - kb0 == min(STAGES, kb1 - kb0)) {  // first item: stage j holds its K block kb0 + j
                        pdl_wait();
                        held = false;
                        for (int j = 0; j <= kb - kb0; ++j) {
                            if (kEarlyB)
                                tma_load_2d(sA + j * A_BYTES, &tmA.m[ab], &S->full[j], (kb0 + j) * KEL, row0);
                            else
                                tma_load_3d(sB + j * B_BYTES, &tmB0, &S->full[j], (kb0 + j) * KEL, n0, expert);
                        }
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
            for (int s = 0; s < STAGES; ++s)
                if ((armed >> s) & 1u)
                    if (!mbar_wait(&S->full[s], (armed_par >> s) & 1u)) record(g.status, MOE_ERR_TIMEOUT);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC = BF16 ? idesc_bf16_f32(BM, BN) : idesc_e4m3_f32(BM, BN);
            int stage = 0, rs = 0, acc = 0;
            uint32_t phase = 0, rphase = 0, aphase = 0;
            bool ok = !(g.stall_test && !mbar_wait(&S->never, 0, g.wait_ns));
            while (ok) {
                if (!mbar_wait(&S->itf[rs], rphase, g.wait_ns)) { ok = false; break; }
                const int item = S->ring[rs];
                mbar_arrive(&S->ite[rs]);
                if (++rs == RING) { rs = 0; rphase ^= 1; }
                if (item < 0) break;
                const int kb0 = (item % ksplit) * KBS, kbn = min(KB, kb0 + KBS) - kb0;
                for (int kb = 0; kb < kbn; ++kb) {
                    if (!mbar_wait(&S->acce[acc], aphase ^ 1, g.wait_ns)) { ok = false; break; }
                    tc_fence_after();
                    if (!mbar_wait(&S->full[stage], phase, g.wait_ns)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t d = tmem + static_cast<uint32_t>(acc * BN);
                    const uint32_t a0 = smem_u32(sA + stage * A_BYTES);
                    const uint32_t b0 = smem_u32(sB + stage * B_BYTES);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {  // 4 x 32 bytes of K: K=32 e4m3 or K=16 bf16 each
                        if (BF16)
                            mma_bf16(d, sw128_kmajor_desc(a0 + k * 32), sw128_kmajor_desc(b0 + k * 32), IDESC, k != 0);
                        else
                            mma_e4m3(d, sw128_kmajor_desc(a0 + k * 32), sw128_kmajor_desc(b0 + k * 32), IDESC, k != 0);
                    }
                    mma_commit(&S->empty[stage]);
                    mma_commit(&S->accf[acc]);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                    if (++acc == 2) { acc = 0; aphase ^= 1; }
                }
            }
            if (!ok) record(g.status, MOE_ERR_TIMEOUT);
            mma_commit(&S->fin);
            if (!mbar_wait(&S->fin, 0)) record(g.status, MOE_ERR_TIMEOUT);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;             // TMEM lane quarter
        const int half = (warp - 2) / 4;    // which 128 accumulator columns
        const int row = q * 32 + lane;
        int rs = 0, acc = 0;
        uint32_t rphase = 0, aphase = 0, xphase = 0;
        int parity = 0;
        for (;;) {
            if (!mbar_wait(&S->itf[rs], rphase, g.wait_ns)) { record(g.status, MOE_ERR_TIMEOUT); break; }
            const int item = S->ring[rs];
            __syncwarp();
            if (lane == 0) mbar_arrive(&S->ite[rs]);
            if (++rs == RING) { rs = 0; rphase ^= 1; }
            if (item < 0) break;
            const int ks = item % ksplit, mn = item / ksplit;
            const int mt = mn / n_tiles, nt = mn - mt * n_tiles;
            const int expert = dense ? 0 : g.tiles[3 * mt];
            const int row0 = dense ? mt * BM : g.tiles[3 * mt + 1];
            const int rows = dense ? min(BM, g.M - row0) : g.tiles[3 * mt + 2];
            const bool row_ok = row < rows;
            const int n0 = nt * BNO;
            const int kb0 = ks * KBS, kbn = min(KB, kb0 + KBS) - kb0;
            // scales: activation row, and the 128-row weight blocks of this thread's columns
            const int nb0 = MODE == 0 ? n0 / 128 : n0 / 128 + half;
            const bool nb_ok = nb0 < NB;
            const float *sa = MODE == 2 ? nullptr : g.sa + (size_t)(row0 + (row_ok ? row : 0)) * KB + kb0;
            const float *sb0 = MODE == 2 ? nullptr : g.sb0 + ((size_t)expert * NB + (nb_ok ? nb0 : 0)) * KB + kb0;
            const float *sb1 = MODE == 0 ? g.sb1 + ((size_t)expert * NB + nb0) * KB + kb0 : sb0;

            float accr[128];
#pragma unroll
            for (int i = 0; i < 128; ++i) accr[i] = 0.0f;
            bool ok = true;
            // the scales of K block kb + 1 are loaded while block kb is promoted
            float na = 0.0f, nb0v = 0.0f, nb1v = 0.0f;
            if (MODE != 2 && kbn > 0) {
                na = row_ok ? sa[0] : 0.0f;
                nb0v = nb_ok ? sb0[0] : 0.0f;
                nb1v = MODE == 0 ? sb1[0] : 0.0f;
            }
            for (int kb = 0; kb < kbn; ++kb) {
                float c0 = 1.0f, c1 = 1.0f;  // mode 2: plain sum of the K-block partials
                if (MODE != 2) {
                    const float a_s = na;
                    c0 = nb_ok ? a_s * nb0v : 0.0f;
                    c1 = MODE == 0 ? a_s * nb1v : c0;
                    if (kb + 1 < kbn) {
                        na = row_ok ? sa[kb + 1] : 0.0f;
                        nb0v = nb_ok ? sb0[kb + 1] : 0.0f;
                        nb1v = MODE == 0 ? sb1[kb + 1] : 0.0f;
                    }
                }
                if (!mbar_wait(&S->accf[acc], aphase, g.wait_ns)) { ok = false; break; }
                tc_fence_after();
                const uint32_t tb = tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * BN);
                // mode 0: chunks 0-3 = gate columns, 4-7 = up columns of this half
                auto chunk_col = [&](int c) {
                    return MODE == 0 ? (c < 4 ? half * 64 + c * 16 : 128 + half * 64 + (c - 4) * 16) : half * 128 + c * 16;
                };
                if (MODE != 2) {
#pragma unroll
                    for (int c = 0; c < 8; c += 2) {  // two loads per TMEM wait
                        uint32_t ra[16], rb[16];
                        tmem_ld16x2_sync(tb + chunk_col(c), tb + chunk_col(c + 1), ra, rb);
                        const float cs = (MODE == 0 && c >= 4) ? c1 : c0;
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            accr[c * 16 + i] = fmaf(cs, __uint_as_float(ra[i]), accr[c * 16 + i]);
                            accr[(c + 1) * 16 + i] = fmaf(cs, __uint_as_float(rb[i]), accr[(c + 1) * 16 + i]);
                        }
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const int col = chunk_col(c);
                        if (n0 + col >= g.N) continue;  // warp-uniform: columns past E
                        uint32_t r[16];
                        tmem_ld16_sync(tb + col, r);
#pragma unroll
                        for (int i = 0; i < 16; ++i) accr[c * 16 + i] = fmaf(c0, __uint_as_float(r[i]), accr[c * 16 + i]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&S->acce[acc]);
                if (++acc == 2) { acc = 0; aphase ^= 1; }
            }
            if (!ok) { record(g.status, MOE_ERR_TIMEOUT); break; }

            if (MODE == 0) {
                // h = silu(gate) * up for this thread's 64 columns, then the 128-column
                // group's amax from both halves, then e4m3 codes and the group scale.
                float m = 0.0f;
#pragma unroll
                for (int i = 0; i < 64; ++i) {
                    accr[i] = silu(accr[i]) * accr[64 + i];
                    m = fmaxf(m, fabsf(accr[i]));
                }
                S->xam[parity][half][row] = m;
                __syncwarp();
                if (lane == 0) mbar_arrive(&S->xbar[q]);
                if (!mbar_wait(&S->xbar[q], xphase, g.wait_ns)) { record(g.status, MOE_ERR_TIMEOUT); break; }
                xphase ^= 1;
                const float amax = fmaxf(S->xam[parity][0][row], S->xam[parity][1][row]);
                parity ^= 1;
                const float sc = amax == 0.0f ? 1.0f : __fdiv_rn(amax, 448.0f);
                const int col = n0 + half * 64;
                if (row_ok && col < g.N) {
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        pk[i] = amax == 0.0f ? 0u
                                             : e4m3_pair(qdiv(accr[4 * i], sc), qdiv(accr[4 * i + 1], sc)) |
                                                   (e4m3_pair(qdiv(accr[4 * i + 2], sc), qdiv(accr[4 * i + 3], sc)) << 16);
                    uint4 *dst = reinterpret_cast<uint4 *>(g.out_q + (size_t)(row0 + row) * g.N + col);
#pragma unroll
                    for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                    if (half == 0) g.out_s[(size_t)(row0 + row) * NB + n0 / 128] = sc;
                }
            } else if (MODE == 2) {
                // partial logits of K split ks: [ksplit][M][N] fp32.  With N a multiple of
                // 4 (rows 16-byte aligned), 16 columns at a time go through the warp's
                // transpose buffer, so that each store covers 64 contiguous bytes of 8 rows
                // (the thread's own row would be 32 scattered 16-byte pieces per store).
                const int col = n0 + half * 128;
                const int total2 = (g.M + BM - 1) / BM * n_tiles * ksplit;
                if ((g.N & 3) == 0 && g.reverse == 2 && item + (int)gridDim.x >= total2) {
                    // The CTA's last item (items are dealt out statically): its last
                    // accumulator wait above means every MMA, and so every read of the
                    // stages, is done, and no further loads come.  The warp writes its 32
                    // rows x 128 columns into the idle stages as four 32 x 32 boxes in the
                    // 128-byte swizzled layout (chunk j of row r at j ^ (r & 7); eight
                    // consecutive rows hit distinct bank groups) and one lane stores them
                    // with the TMA, which clips rows past M and columns past N.
                    uint8_t *box0 = sA + (size_t)(warp - 2) * 4 * 4096;  // 8 warps x 16 KB
#pragma unroll
                    for (int b = 0; b < 4; ++b) {
                        if (col + 32 * b >= g.N) break;  // warp-uniform
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            *reinterpret_cast<float4 *>(box0 + b * 4096 + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                                make_float4(accr[32 * b + 4 * j], accr[32 * b + 4 * j + 1], accr[32 * b + 4 * j + 2],
                                            accr[32 * b + 4 * j + 3]);
                    }
                    fence_proxy_async_shared_cta();
                    __syncwarp();
                    if (lane == 0) {
                        for (int b = 0; b < 4 && col + 32 * b < g.N; ++b)
                            tma_store_3d(&tmB1, box0 + b * 4096, col + 32 * b, row0 + q * 32, ks);
                        bulk_commit_group();
                        bulk_wait_all();
                    }
                    __syncwarp();
                } else if ((g.N & 3) == 0) {
                    float *buf = reinterpret_cast<float *>(sB + STAGES * B_BYTES + EPI2_OFF) +
                                 (warp - 2) * 32 * EPI2_ROW;
                    const int rr = lane % 8, m = lane / 8;  // read-back: row rr + 8p, 16-byte piece m
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        if (col + 16 * c >= g.N) break;  // warp-uniform: columns past N
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            reinterpret_cast<float4 *>(buf + lane * EPI2_ROW)[i] =
                                make_float4(accr[16 * c + 4 * i], accr[16 * c + 4 * i + 1], accr[16 * c + 4 * i + 2],
                                            accr[16 * c + 4 * i + 3]);
                        __syncwarp();
#pragma unroll
                        for (int p = 0; p < 4; ++p) {
                            const int r = 8 * p + rr;  // row within the warp's 32
                            const float4 v = reinterpret_cast<const float4 *>(buf + r * EPI2_ROW)[m];
                            const int cc = col + 16 * c + 4 * m;
                            if (q * 32 + r < rows && cc < g.N)
                                *reinterpret_cast<float4 *>(g.out_f32 + ((size_t)ks * g.M + row0 + q * 32 + r) * g.N + cc) = v;
                        }
                        __syncwarp();
                    }
                } else if (row_ok && col < g.N) {
                    float *dst = g.out_f32 + ((size_t)ks * g.M + row0 + row) * g.N + col;
#pragma unroll
                    for (int i = 0; i < 128; ++i)
                        if (col + i < g.N) dst[i] = accr[i];
                }
            } else {
                const int col = n0 + half * 128;
                if (row_ok && col < g.N) {
                    const int flat = g.row_map[row0 + row];
                    uint4 *dst = reinterpret_cast<uint4 *>(g.out + (size_t)flat * g.N + col);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        __nv_bfloat162 v[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) v[j] = __floats2bfloat162_rn(accr[8 * i + 2 * j], accr[8 * i + 2 * j + 1]);
                        dst[i] = *reinterpret_cast<uint4 *>(v);
                    }
                }
                if (COMB)  // both halves of a row arrive (comb_target = 2k), empty ones too
                    combine_arrive(g.out, g.comb_gate, g.comb_out, g.comb_cnt, g.comb_k, g.comb_target, g.N, n_tiles,
                                   nt, row_ok, row_ok ? g.row_map[row0 + row] : 0, lane);
            }
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

bool fp8_smem_attr_ready(int v)  // v: 0 gate/up, 1 down, 2 router logits, 3 down with the fused combine
{
    static std::mutex mu;
    static uint64_t done[4] = {0, 0, 0, 0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    std::lock_guard<std::mutex> lk(mu);
    if (done[v] >> dev & 1ull) return true;
    const int a = (int)smem8_bytes(v);
    cudaError_t e = v == 0   ? cudaFuncSetAttribute(grouped_gemm_fp8_kernel<0, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, a)
                  : v == 1 ? cudaFuncSetAttribute(grouped_gemm_fp8_kernel<1, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, a)
                  : v == 2 ? cudaFuncSetAttribute(grouped_gemm_fp8_kernel<2, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, a)
                           : cudaFuncSetAttribute(grouped_gemm_fp8_kernel<1, false, true>,
                                                  cudaFuncAttributeMaxDynamicSharedMemorySize, a);
    if (e != cudaSuccess) return false;
    done[v] |= 1ull << dev;
    return true;
}

}  // namespace

cudaError_t launch_quantize_rows(const __nv_bfloat16 *src, const int32_t *map, int k, int R, int K, uint8_t *q,
                                 float *s, cudaStream_t st)
{
    const long warps = (long)R * ((K / 128 + 7) / 8);
    return launch_pdl(quantize_rows_kernel, dim3((unsigned)((warps + 7) / 8)), dim3(256), 0, st, src, map, k, R, K, q,
                      s);
}

cudaError_t launch_gather_rows_fp8(const uint8_t *xq, const float *xq_s, const int32_t *s2f, int A, int K, int k,
                                   uint8_t *xs, float *xs_s, cudaStream_t st)
{
    const int rows_per_block = 8;
    return launch_pdl(gather_rows_fp8_kernel, dim3((A + rows_per_block - 1) / rows_per_block),
                      dim3(rows_per_block * 32), 0, st, xq, xq_s, s2f, A, K, k, xs, xs_s);
}

cudaError_t launch_grouped_gemm_fp8(const Fp8GemmArgs &g, const AMaps &tmA, const CUtensorMap &tmB0,
                                    const CUtensorMap &tmB1, cudaStream_t st)
{
    const int grid = g.ctas > 0 ? g.ctas : num_sms();
    const bool comb = g.mode == 1 && g.comb_cnt != nullptr;
    if (!fp8_smem_attr_ready(comb ? 3 : g.mode)) return cudaErrorInvalidValue;
    cudaError_t e;
    if (g.mode == 0)
        e = launch_pdl(grouped_gemm_fp8_kernel<0, false>, dim3(grid), dim3(THREADS), SMEM8, st, tmA, tmB0, tmB1, g);
    else if (comb)  // the combine's code is compiled in only here: it costs the epilogue registers
        e = launch_pdl(grouped_gemm_fp8_kernel<1, false, true>, dim3(grid), dim3(THREADS), SMEM8, st, tmA, tmB0, tmB1,
                       g);
    else if (g.mode == 1)
        e = launch_pdl(grouped_gemm_fp8_kernel<1, false>, dim3(grid), dim3(THREADS), SMEM8, st, tmA, tmB0, tmB1, g);
    else
        e = launch_pdl(grouped_gemm_fp8_kernel<2, true>, dim3(grid), dim3(THREADS), smem8_bytes(2), st, tmA, tmB0,
                       tmB1, g);
    return e;
}

}  // namespace moe
