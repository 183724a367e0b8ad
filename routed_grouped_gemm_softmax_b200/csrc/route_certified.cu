// route_certified.cu -- the router for batches of more than 32 tokens: tensor-core
// logits, certified against the fp32 chain that defines the routing.
//
// The router's logit is the fp32 FMA chain over h ascending (route.cu states the
// contract).  Evaluating all T*E chains costs 2*T*H*E CUDA-core flops, so for large
// batches the chain is evaluated only where it can change the answer:
//  1. router_prep_kernel transposes router_w to [E, H] and takes partial squared
//     column norms (per 256 rows), summed per expert by the certify kernel;
//  2. Lt = x . Wr on the tensor cores (fp8.cu, mode 2: bf16 in, each 64-wide K
//     block summed out of TMEM in fp32, K split over a few slices);
//  3. router_certify_kernel, a CTA per block of tokens:
//     a. per token (a warp), a bound |chain - Lt| <= d_e: the chain's own rounding
//        is at most H u sum_h |x_h w_he| (u = 2^-24, recursive summation with fma),
//        the tensor-core value's at most (64 * 4u + (H/64 + slices) u) times the
//        same sum (each 64-term block accumulated within 4 ulps, then one rounding
//        per block and slice sum); sum_h |x_h w_he| <= |x_t| |w_e| (Cauchy-Schwarz);
//        1% margin, plus a few ulps of the bias add and of the values themselves.
//        tau = the k-th largest lower bound Lt - d; an expert whose upper bound
//        Lt + d is below tau has k experts strictly above it and cannot be chosen.
//        The others -- the k chosen plus near-ties -- are the token's candidates;
//     b. the exact chain of every candidate of the block: the block's x rows and
//        its slice of router_w^T stream through shared memory in chunks of up to
//        512 values of h (tensor-map tiles, two or three stages on mbarriers), a
//        thread running one chain per round with the mixed-precision chain step;
//        each exact value is checked against its bound (a miss records
//        MOE_ERR_ROUTER_BOUND);
//     c. per token (a warp), top-k and softmax on the candidates' exact values.
// The chosen experts and gates are therefore those of the chain definition.
#include <atomic>
#include <cfloat>
#include <climits>

#include "moe_internal.h"
#include "pdl.cuh"
#include "route_common.cuh"
#include "sm100_ptx.cuh"

namespace moe {

// The staging policy set by moe_set_cert_staging (moe_api.cu): {max stages, min stages,
// max boxes per chunk}, each 0 for the default (3, 2, 8).
void cert_staging(int *max_stages, int *min_stages, int *max_boxes);

namespace {

constexpr int kPrepE = 16;     // experts per CTA of router_prep_kernel
constexpr int kPrepH = 256;    // h rows per CTA

// Wr [H, E] -> wrt [E, H] (one 256 x 16 tile per CTA), and the partial squared
// column norms wsq_part[h / 256][e] = sum over the tile's rows of Wr[h, e]^2 (fp32;
// the bound inflates it).
__global__ void __launch_bounds__(256) router_prep_kernel(const __nv_bfloat16 *__restrict__ wr, int H, int E,
                                                          __nv_bfloat16 *__restrict__ wrt,
                                                          float *__restrict__ wsq_part)
{
    pdl_wait();
    pdl_trigger();
    __shared__ uint16_t tile[kPrepH][kPrepE + 2];
    const int tid = threadIdx.x;
    const int e0 = blockIdx.x * kPrepE, h0 = blockIdx.y * kPrepH;
    const uint16_t *w16 = reinterpret_cast<const uint16_t *>(wr);
    uint16_t *o16 = reinterpret_cast<uint16_t *>(wrt);
    {
        constexpr int kSteps = kPrepH / (256 / kPrepE);  // 16 threads per row, all loads in flight together
        uint16_t v[kSteps];
        const int e = e0 + tid % kPrepE;
#pragma unroll
        for (int i = 0; i < kSteps; ++i) {
            const int h = h0 + tid / kPrepE + i * (256 / kPrepE);
            v[i] = (h < H && e < E) ? w16[(size_t)h * E + e] : uint16_t(0);
        }
#pragma unroll
        for (int i = 0; i < kSteps; ++i) tile[tid / kPrepE + i * (256 / kPrepE)][tid % kPrepE] = v[i];
    }
    __syncthreads();
    // thread (el, part): rows r = part mod 16 of expert el, then a 16-lane tree
    const int el = tid / 16, part = tid % 16;
    float ss = 0.0f;
    for (int r = part; r < kPrepH; r += 16) {
        const float f = __uint_as_float(static_cast<uint32_t>(tile[r][el]) << 16);
        ss = fmaf(f, f, ss);
    }
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if (part == 0 && e0 + el < E) wsq_part[(size_t)blockIdx.y * E + e0 + el] = ss;
    for (int v = tid; v < kPrepE * kPrepH; v += 256) {  // 16 expert rows of 256 values
        const int ee = v / kPrepH, r = v % kPrepH;
        const int h = h0 + r, e = e0 + ee;
        if (h < H && e < E) o16[(size_t)e * H + h] = tile[r][ee];
    }
}

// Threads of a certify CTA: 1024 (a chain each, 64 registers) up to 256 experts, 512
// above (the per-lane arrays of 512 or more experts need the registers).
constexpr int kCertWarps = 32;  // the most warps a CTA has (sizes the per-warp scratch)
__host__ __device__ constexpr int cert_threads(int maxv) { return maxv <= 8 ? 1024 : 512; }
constexpr int kCertMaxStages = 8;  // staging barriers (the policy's cap, 3 by default)
constexpr int kCertMaxTB = 128;  // tokens per block
constexpr int kCertSmem = 227 * 1024;

struct CertifyArgs {
    const float *lt;        // [ksplit, T, E] partial tensor-core logits
    float *ex;              // = lt slice 0: receives the exact values of the chosen experts
    int ksplit;
    const __nv_bfloat16 *x;
    const float *wsq_part, *bias;  // wsq_part [nparts, E]
    int nparts;
    int T, H, E, k;
    int TB;                 // tokens of a block: the tokens of one cluster of CTAs
    int EB;                 // experts of a CTA's slice: CTA r of a cluster runs the chains of experts r*EB ..
    float eps;
    int32_t *ncand;         // [T] candidates per token
    RouterCand *list;       // [T, E] the candidates of token t in slots t*E .. t*E + ncand[t] - 1, ascending e;
                            // after the chains, .v holds the exact value
    int32_t *idx;
    float *gate;
    int32_t *status;
    float *audit_v, *audit_d;  // null, or [T, E]: every tensor-core logit and its bound
    int xrows;              // rows of an x tile (TB rounded up to 8)
    int erows;              // staged router rows (EB rounded up to 8, or to 256 above 256)
    int ebox;               // rows of one router tile (<= 256)
    int nbx;                // 64-column tiles per chunk
    int stages;             // 1..kCertMaxStages
    int stage_bytes;        // nbx * (xrows + erows) * 128
};

// Fixed part of the dynamic shared memory: the stage barriers, per-token counts,
// first chains and prefix, expert norms, per-warp top-k outputs; the stages follow at
// a 1024-byte boundary (the 128-byte swizzle repeats every 8 rows of 128 bytes).
__host__ __device__ inline size_t cert_fixed_bytes(int E, int k)
{
    const size_t words = (size_t)3 * kCertMaxTB + (kCertMaxTB + 1) + E + 8 + (size_t)2 * kCertWarps * k;
    return (kCertMaxStages * 8 + words * 4 + 1023) / 1024 * 1024;
}

__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_nctarank()
{
    uint32_t n;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(n));
    return n;
}
// Every thread of every CTA of the cluster arrives; this CTA's threads wait, and the
// global and shared writes made before the arrival are visible after the wait.  A
// cluster of one CTA is a plain CTA barrier.
__device__ __forceinline__ void cluster_barrier(uint32_t csize)
{
    if (csize == 1) {
        __syncthreads();
        return;
    }
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// 16-byte chunk j (0..7) of row r of a 128-byte-swizzled tile.
__device__ __forceinline__ const uint4 *sw128_chunk(const uint8_t *tile, int r, int j)
{
    return reinterpret_cast<const uint4 *>(tile + r * 128 + ((j ^ (r & 7)) << 4));
}

template <int MAXV, int NT = cert_threads(MAXV)>
__global__ void __launch_bounds__(NT)
    router_certify_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                          const CertifyArgs a)
{
    extern __shared__ __align__(128) uint8_t csm[];
    constexpr int NW = NT / 32;
    const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
    const int E = a.E, H = a.H, k = a.k;
    // the cluster's block of tokens; this CTA's slice of the experts, and its share of
    // the block's tokens in the per-token phases (tokens r, r + C, ...)
    const uint32_t C = cluster_nctarank(), rank = cluster_ctarank();
    const int t0 = (int)(blockIdx.x / C) * a.TB;
    const int tb = max(0, min(a.TB, a.T - t0));
    const int eb0 = min(E, (int)rank * a.EB), eb1 = min(E, eb0 + a.EB);
    uint64_t *full = reinterpret_cast<uint64_t *>(csm);        // [kCertMaxStages] staging barriers
    int *nc = reinterpret_cast<int *>(full + kCertMaxStages);  // [kCertMaxTB] candidates of the tokens of this CTA
    int *clo = nc + kCertMaxTB;                                 // [kCertMaxTB] first candidate in the slice
    int *cnt = clo + kCertMaxTB;                                // [kCertMaxTB] candidates in the slice
    int *cb = cnt + kCertMaxTB;                                 // [kCertMaxTB + 1] chain prefix over tokens
    float *wn = reinterpret_cast<float *>(cb + kCertMaxTB + 1);  // [E] norms of the router columns
    int *misc = reinterpret_cast<int *>(wn + E);                // [8]: 1 chains
    int *wse = misc + 8;                                        // [warps][k]
    float *wsv = reinterpret_cast<float *>(wse + kCertWarps * k);  // [warps][k]
    // stages at a 1024-byte boundary of the shared address space (the launch adds 1 KB of slack)
    const uint32_t fixed_end = smem_u32(csm) + (uint32_t)cert_fixed_bytes(E, k);
    uint8_t *stage0 = csm + (((fixed_end + 1023u) & ~1023u) - smem_u32(csm));

    // A chunk is nbx 64-column blocks of h (nbx divides H / 64): the block's x rows of
    // each, then the router rows of the CTA's experts (router_w^T) of each, stored
    // [nbx][xrows][128 B] and [erows / ebox][nbx][ebox][128 B], every block with the
    // 128-byte swizzle so that eight lanes reading the same 16-byte column of eight
    // rows hit eight bank groups when the rows differ mod 8.  One TMA box brings all nbx
    // blocks of the x rows and one each ebox router rows: the SM's TMA throughput
    // grows with the bytes behind each box and each barrier.  Chunk g (a running count
    // over rounds) lives in stage g % stages and completes on full[g % stages].
    const int S = a.stages, hc = a.nbx * 64, nch = H / hc;
    const size_t x_bytes = (size_t)a.nbx * a.xrows * 128;
    auto issue = [&](int ch, uint32_t g) {  // thread 0
        uint8_t *st = stage0 + (size_t)(g % S) * a.stage_bytes;
        mbar_arrive_expect_tx(&full[g % S], (uint32_t)a.stage_bytes);
        tma_load_3d(st, &tm_x, &full[g % S], 0, t0, ch * a.nbx);
        for (int r = 0; r < a.erows; r += a.ebox)
            tma_load_3d(st + x_bytes + (size_t)r * a.nbx * 128, &tm_w, &full[g % S], 0, eb0 + r, ch * a.nbx);
    };

    if (tid == 0) {
        for (int s = 0; s < kCertMaxStages; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    __syncthreads();
    pdl_wait();
    pdl_trigger();
    // The first round's first chunks depend on nothing below: their copies overlap the
    // bounds.  Every chain round consumes all nch chunks, and a block has at least k
    // chains, so each of these copies is waited for before the kernel ends.
    if (tid == 0)
        for (int ch = 0; ch < min(S, nch); ++ch) issue(ch, ch);
    for (int e = tid; e < E; e += NT) {
        float q = 0.0f;
        for (int j = 0; j < a.nparts; ++j) q += a.wsq_part[(size_t)j * E + e];
        wn[e] = sqrtf(q);
    }
    __syncthreads();

    // ---- a. bounds and candidates, a warp per token; the token's loads (bias, the
    // logit slices, its x row) are all issued before the first is used
    for (int tl = (int)rank + (int)C * warp; tl < tb; tl += (int)C * NW) {
        const int t = t0 + tl;
        float bias[MAXV], v[MAXV];
#pragma unroll
        for (int i = 0; i < MAXV; ++i) {
            const int e = lane + 32 * i;
            bias[i] = (a.bias && e < E) ? a.bias[e] : 0.0f;
            v[i] = 0.0f;
        }
#pragma unroll
        for (int q = 0; q < kRouterKSplitMax; ++q) {  // slices summed in order
            if (q < a.ksplit) {
                const float *row = a.lt + ((size_t)q * a.T + t) * E;
#pragma unroll
                for (int i = 0; i < MAXV; ++i) {
                    const int e = lane + 32 * i;
                    if (e < E) v[i] += row[e];
                }
            }
        }
        float ss = 0.0f;
        const uint4 *xr = reinterpret_cast<const uint4 *>(a.x + (size_t)t * H);
#pragma unroll 8
        for (int h8 = lane; h8 < H / 8; h8 += 32) {
            const uint4 q = xr[h8];
            const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float lo = __uint_as_float(w4[i] << 16), hi = __uint_as_float(w4[i] & 0xFFFF0000u);
                ss = fmaf(lo, lo, ss);
                ss = fmaf(hi, hi, ss);
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const float xn = sqrtf(ss) * 1.001f;
        // the slices' sum, then the bias
        uint32_t key[MAXV];
        float lo[MAXV];
#pragma unroll
        for (int i = 0; i < MAXV; ++i) {
            const int e = lane + 32 * i;
            float s = v[i];
            if (a.bias) s += bias[i];
            v[i] = e < E ? s : -INFINITY;
            const float d = e < E ? a.eps * xn * wn[e] * 1.001f + fabsf(s) * 4.8e-7f + 1e-30f : 0.0f;
            lo[i] = e < E ? s - d : 0.0f;
            key[i] = e < E ? order_key(lo[i]) : 0u;
            if (a.audit_v && e < E) {
                a.audit_v[(size_t)t * E + e] = s;
                a.audit_d[(size_t)t * E + e] = d;
            }
        }
        // tau: the k-th largest lower bound
        warp_topk<MAXV>(key, lo, k, wse + warp * k, wsv + warp * k);
        const float tau = wsv[warp * k + k - 1];
        // candidates (upper bound >= tau), ascending expert index
        RouterCand *out = a.list + (size_t)t * E;
        int pos = 0;
#pragma unroll
        for (int i = 0; i < MAXV; ++i) {
            const int e = lane + 32 * i;
            const float d = v[i] - lo[i];
            const bool c = e < E && v[i] + d >= tau;
            const unsigned m = __ballot_sync(0xffffffffu, c);
            if (c) out[pos + __popc(m & ((1u << lane) - 1u))] = RouterCand{t, e, v[i], d};
            pos += __popc(m);
        }
        if (lane == 0) {
            nc[tl] = pos;
            a.ncand[t] = pos;
        }
        __syncwarp();
    }
    cluster_barrier(C);  // every token's candidates listed

    // this CTA's chains: the candidates of the block's tokens in its expert slice (a
    // contiguous run of each token's list, which ascends by expert)
    for (int tl = warp; tl < tb; tl += NW) {
        const int t = t0 + tl;
        int lo = 0, n = 0;
        if (C == 1) {
            n = nc[tl];
        } else {
            const int m = a.ncand[t];
            const RouterCand *cl = a.list + (size_t)t * E;
            int hi = 0;
            for (int p = lane; p - lane < m; p += 32) {
                const int e = p < m ? cl[p].e : INT_MAX;
                lo += __popc(__ballot_sync(0xffffffffu, e < eb0));
                hi += __popc(__ballot_sync(0xffffffffu, e < eb1));
            }
            n = hi - lo;
        }
        if (lane == 0) {
            clo[tl] = lo;
            cnt[tl] = n;
        }
    }
    __syncthreads();
    // chain prefix over the block's tokens (tb <= 128: four tokens per lane)
    if (warp == 0) {
        int c4[4], sum = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int tl = 4 * lane + i;
            c4[i] = tl < tb ? cnt[tl] : 0;
            sum += c4[i];
        }
        int inc = sum;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, inc, off);
            if (lane >= off) inc += o;
        }
        int run = inc - sum;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            cb[4 * lane + i] = run;
            run += c4[i];
        }
        if (lane == 31) {
            cb[kCertMaxTB] = inc;
            misc[1] = inc;
        }
    }
    __syncthreads();
    const int nchain = misc[1];

    // ---- b. exact chains of the candidates, one per thread and round; one CTA barrier
    // per chunk frees its stage for the refill
    // (at least one round, so that the chunks issued before the bounds are read even by
    // a CTA whose expert slice holds no candidate)
    uint32_t g0 = 0;
    bool failed = false;
    for (int r0 = 0; r0 == 0 || r0 < nchain; r0 += NT) {
        const int c = r0 + tid;
        const bool on = c < nchain;
        int ctl = 0, cpos = 0;
        RouterCand cc{0, 0, 0.0f, 0.0f};
        float acc = 0.0f;
        if (on) {
            int lo = 0, hi = tb;  // largest tl with cb[tl] <= c
            while (hi - lo > 1) {
                const int mid = (lo + hi) / 2;
                if (cb[mid] <= c) lo = mid;
                else hi = mid;
            }
            ctl = lo;
            cpos = clo[lo] + c - cb[lo];
            cc = a.list[(size_t)(t0 + lo) * E + cpos];
        }
        if (tid == 0 && r0 > 0)
            for (int ch = 0; ch < min(S, nch); ++ch) issue(ch, g0 + ch);
        for (int ch = 0; ch < nch; ++ch) {
            const uint32_t g = g0 + ch;
            if (!mbar_wait(&full[g % S], (g / S) & 1u, failed ? 1000000ull : kWaitLimitNs)) {
                failed = true;
                atomicCAS(a.status, 0, MOE_ERR_TIMEOUT);
            }
            const uint8_t *st = stage0 + (size_t)(g % S) * a.stage_bytes;
            if (on) {
                // the chain's router row: block (el / ebox) of the router part, row el % ebox
                const int el = cc.e - eb0;
                const uint8_t *wr0 = st + x_bytes + (size_t)(el / a.ebox) * a.nbx * a.ebox * 128;
                for (int b = 0; b < a.nbx; ++b) {
                    const uint8_t *xt = st + (size_t)b * a.xrows * 128;
                    const uint8_t *wt = wr0 + (size_t)b * a.ebox * 128;
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        acc = chain_step8(*sw128_chunk(xt, ctl, j), *sw128_chunk(wt, el % a.ebox, j), acc);
                }
            }
            __syncthreads();  // stage g % S consumed by every thread
            if (tid == 0 && ch + S < nch) issue(ch + S, g + S);
        }
        g0 += nch;
        if (on) {
            float v = acc;
            if (a.bias) v = __fadd_rn(v, a.bias[cc.e]);
            a.list[(size_t)(t0 + ctl) * E + cpos].v = v;
            if (!(fabsf(v - cc.v) <= cc.d)) atomicCAS(a.status, 0, MOE_ERR_ROUTER_BOUND);
        }
    }
    cluster_barrier(C);  // every exact value written

    // ---- c. top-k (larger exact value first, lower index on ties) and softmax; a
    // token with at most 32 candidates holds one per lane
    for (int tl = (int)rank + (int)C * warp; tl < tb; tl += (int)C * NW) {
        const int t = t0 + tl;
        const int n = nc[tl];
        const RouterCand *cl = a.list + (size_t)t * E;
        int *se = wse + warp * k;
        float *sv = wsv + warp * k;
        if (n <= 32) {
            RouterCand c{0, 0, 0.0f, 0.0f};
            if (lane < n) c = cl[lane];
            uint32_t key1[1] = {lane < n ? order_key(c.v) : 0u};
            const float val1[1] = {c.v};
            warp_topk<1>(key1, val1, k, se, sv);
            for (int j = 0; j < k; ++j) {
                const int e = __shfl_sync(0xffffffffu, c.e, se[j] & 31);
                if (lane == 0) {
                    a.idx[(size_t)t * k + j] = e;
                    a.ex[(size_t)t * E + e] = sv[j];
                }
            }
        } else {
            uint32_t key[MAXV];
            float val[MAXV];
            int ce[MAXV];
#pragma unroll
            for (int i = 0; i < MAXV; ++i) {
                const int p = lane + 32 * i;  // candidates are in ascending expert order
                RouterCand c{0, 0, 0.0f, 0.0f};
                if (p < n) c = cl[p];
                ce[i] = c.e;
                val[i] = c.v;
                key[i] = p < n ? order_key(c.v) : 0u;
            }
            warp_topk<MAXV>(key, val, k, se, sv);
            // slot -> expert: the slot order is the expert order, so the tie rule holds
            for (int j = 0; j < k; ++j) {
                const int p = se[j];
                int mine = 0;
#pragma unroll
                for (int i = 0; i < MAXV; ++i)
                    if (i == (p >> 5)) mine = ce[i];
                const int e = __shfl_sync(0xffffffffu, mine, p & 31);
                if (lane == 0) {
                    a.idx[(size_t)t * k + j] = e;
                    a.ex[(size_t)t * E + e] = sv[j];
                }
            }
        }
        const float m = sv[0];
        float s = 0.0f;
        for (int j = lane; j < k; j += 32) s += expf(sv[j] - m);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        for (int j = lane; j < k; j += 32) a.gate[(size_t)t * k + j] = expf(sv[j] - m) / s;
        __syncwarp();
    }
}

// Launch with C CTAs per cluster (the expert slices of one token block) and
// programmatic stream serialisation.
template <int MAXV>
cudaError_t launch_certify(const CUtensorMap &tm_x, const CUtensorMap &tm_w, const CertifyArgs &a, int grid, int C,
                           cudaStream_t st)
{
    auto kern = router_certify_kernel<MAXV>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kCertSmem);
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)C;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(cert_threads(MAXV));
    cfg.dynamicSmemBytes = kCertSmem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, tm_x, tm_w, a);
}

// How many clusters of C certify CTAs can be resident at once (0 if none, or if the
// query fails); C = 1 is one CTA per SM.  Queried once per (kernel, C).
template <int MAXV>
int cert_clusters(int C)
{
    static std::atomic<int> cached[4] = {-1, -1, -1, -1};
    const int slot = C == 1 ? 0 : C == 2 ? 1 : C == 4 ? 2 : 3;
    int v = cached[slot].load();
    if (v >= 0) return v;
    if (C == 1) {
        v = num_sms();
    } else {
        auto kern = router_certify_kernel<MAXV>;
        v = 0;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kCertSmem) == cudaSuccess) {
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = (unsigned)C;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cudaLaunchConfig_t cfg{};
            cfg.gridDim = dim3((unsigned)C);
            cfg.blockDim = dim3(cert_threads(MAXV));
            cfg.dynamicSmemBytes = kCertSmem;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess) v = n;
            else (void)cudaGetLastError();
        }
    }
    cached[slot].store(v);
    return v;
}

// The certify launch for T tokens: tokens in blocks of TB, one cluster of C CTAs per
// block, CTA r of a cluster taking the chains of experts r*EB .. (r+1)*EB - 1.  C is
// the cluster size (1, 2, 4 or 8 that fit) whose CTAs stage the fewest rows per chunk
// (the block's x rows plus the slice's router rows): fewer rows leave room for wider
// chunks, each chunk costs the chain phase a CTA barrier and a pipeline restart, and
// the per-token phases take T / (resident CTAs) tokens per CTA either way.
template <int MAXV>
cudaError_t certify_shape_and_launch(const __nv_bfloat16 *x, const __nv_bfloat16 *wrt, CertifyArgs a, int T, int E,
                                     int k, cudaStream_t st)
{
    int bestC = 0, bestTB = 0, bestCost = INT_MAX;
    for (int C : {1, 2, 4, 8}) {
        if (C > 1 && E < 16 * C) break;  // slices of fewer than 16 experts stage little less
        const int clusters = cert_clusters<MAXV>(C);
        if (clusters < 1) continue;
        const int TB = (T + clusters - 1) / clusters;
        if (TB > kCertMaxTB) continue;
        const int EB = (E + C - 1) / C;
        const int cost = (TB + 7) / 8 * 8 + (EB <= 256 ? (EB + 7) / 8 * 8 : (EB + 255) / 256 * 256);
        if (cost < bestCost) {
            bestCost = cost;
            bestC = C;
            bestTB = TB;
        }
    }
    if (bestC == 0) {  // more tokens than the resident CTAs take in blocks of kCertMaxTB
        bestC = 1;
        bestTB = kCertMaxTB;
    }
    const int C = bestC, TB = bestTB, EB = (E + C - 1) / C;
    const int xrows = (TB + 7) / 8 * 8;
    const int erows = EB <= 256 ? (EB + 7) / 8 * 8 : (EB + 255) / 256 * 256;
    const int ebox = erows < 256 ? erows : 256;
    const size_t room = (size_t)kCertSmem - 1024 - cert_fixed_bytes(E, k);
    int max_st = 0, min_st = 0, max_nbx = 0;  // the staging policy (moe_set_cert_staging)
    cert_staging(&max_st, &min_st, &max_nbx);
    max_st = max_st > 0 ? max_st : 3;
    min_st = min_st > 0 ? min_st : 2;
    int nbx = max_nbx > 0 ? max_nbx : 8, stages = 0;
    for (; nbx >= 1; nbx /= 2) {  // the widest chunk dividing H that still leaves min_st stages
        if ((a.H / 64) % nbx) continue;
        stages = (int)(room / ((size_t)nbx * (xrows + erows) * 128));
        if (stages >= min_st || nbx == 1) break;
    }
    if (stages > max_st) stages = max_st;
    if (stages > kCertMaxStages) stages = kCertMaxStages;
    if (stages < 1) return cudaErrorInvalidValue;
    CUtensorMap tm_x, tm_w;
    if (!encode_sw128_chunked_bf16(&tm_x, x, T, a.H, xrows, nbx) ||
        !encode_sw128_chunked_bf16(&tm_w, wrt, E, a.H, ebox, nbx))
        return cudaErrorInvalidValue;
    a.TB = TB;
    a.EB = EB;
    a.xrows = xrows;
    a.erows = erows;
    a.ebox = ebox;
    a.nbx = nbx;
    a.stages = stages;
    a.stage_bytes = nbx * (xrows + erows) * 128;
    const int grid = (T + TB - 1) / TB * C;
    return launch_certify<MAXV>(tm_x, tm_w, a, grid, C, st);
}

}  // namespace

cudaError_t launch_route_certified(const moe_dims_t &d, const __nv_bfloat16 *x, const __nv_bfloat16 *wr,
                                   const float *bias, float *logits, int32_t *idx, float *gate,
                                   const RouterScratch &rs, WsHeader *hdr, cudaStream_t st)
{
    const int T = d.T, H = d.H, E = d.E, k = d.top_k;
    const int nparts = (H + kPrepH - 1) / kPrepH;
    cudaError_t e = launch_pdl(router_prep_kernel, dim3((E + kPrepE - 1) / kPrepE, nparts), dim3(256), 0, st, wr, H,
                               E, rs.wrt, rs.wsq);
    if (e != cudaSuccess) return e;
    int ks = 1;
    if ((e = tc_router_logits(x, rs.wrt, T, H, E, logits, hdr, &ks, st)) != cudaSuccess) return e;
    const float u = 5.9604644775390625e-08f;  // 2^-24
    const float eps = ((float)H * u + 256.0f * u + (float)(H / 64 + ks) * u) * 1.01f;
    CertifyArgs a{logits, logits, ks, x, rs.wsq, bias, nparts, T, H, E, k, 0, 0, eps, rs.ncand, rs.list,
                  idx, gate, &hdr->status, rs.audit_v, rs.audit_d, 0, 0, 0, 0, 0, 0};
    const int vpl = (E + 31) / 32;
    if (vpl <= 1) return certify_shape_and_launch<1>(x, rs.wrt, a, T, E, k, st);
    if (vpl <= 2) return certify_shape_and_launch<2>(x, rs.wrt, a, T, E, k, st);
    if (vpl <= 4) return certify_shape_and_launch<4>(x, rs.wrt, a, T, E, k, st);
    if (vpl <= 8) return certify_shape_and_launch<8>(x, rs.wrt, a, T, E, k, st);
    if (vpl <= 16) return certify_shape_and_launch<16>(x, rs.wrt, a, T, E, k, st);
    return certify_shape_and_launch<32>(x, rs.wrt, a, T, E, k, st);
}

}  // namespace moe
