// route.cu -- router logits and softmax top-k gating for small batches, and the
// router's dispatch.
//
// The router picks, for every token, the top-k experts by router logit and
// weights their outputs by a softmax over the chosen k (vLLM fused-MoE page,
// section 02; the Weave review, section 1.1, describes the same top-k router).
//
// Logit contract: logit[t,e] is the fp32 result of the fused-multiply-add chain
// over h = 0..H-1 in ascending order starting from 0.0f, followed by one fp32
// addition of bias[e].  Every chain evaluated here runs in exactly that order on
// one thread, so the logits -- and the integer routing decision taken on them --
// are reproducible bit for bit.
//
// T <= 32: every (t,e) chain on the CUDA cores (route_logits_small_kernel, or the
//   tiled route_logits_kernel for shapes it does not take), then top-k + softmax
//   with one warp per token (route_topk_kernel), or top-k + softmax + the stable
//   grouping by expert in one CTA (topk_permute_small_kernel) inside the forward.
// T > 32: tensor-core logits certified against the chains (route_certified.cu).
#include <cfloat>
#include <climits>

#include "moe_internal.h"
#include "pdl.cuh"
#include "route_common.cuh"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

// Logits tile kernel.  A CTA owns TT tokens x TE experts, a thread RT x RE of them.
// The h axis is walked in chunks of HC: the chunk after the current one is fetched
// from global memory into registers (bf16) while the current one -- already in
// shared memory as fp32, x transposed to [h][token] so a thread's tokens are
// contiguous -- feeds the FMA chains; one barrier per chunk.
template <int TT, int TE, int RT, int RE, int HC>
struct LogitsTile {
    static constexpr int NX = TE / RE;             // threads along experts
    static constexpr int NT = (TT / RT) * NX;      // threads per CTA
    static constexpr int XV = TT * HC / 8;         // 16-byte vectors of an x chunk
    static constexpr int WV = HC * TE / 8;         // 16-byte vectors of a router_w chunk
    static constexpr int XPT = (XV + NT - 1) / NT; // x vectors per thread
    static constexpr int WPT = (WV + NT - 1) / NT; // w vectors per thread
    static constexpr int SMEM_FLOATS = 2 * HC * (TT + TE);
};

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &v, float (&f)[8])
{
    const __nv_bfloat162 *p = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 t = __bfloat1622float2(p[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}

template <int TT, int TE, int RT, int RE, int HC>
__global__ void __launch_bounds__(LogitsTile<TT, TE, RT, RE, HC>::NT)
route_logits_kernel(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ wr,
                    const float *__restrict__ bias, int T, int H, int E, float *__restrict__ logits)
{
    pdl_wait();
    pdl_trigger();
    using L = LogitsTile<TT, TE, RT, RE, HC>;
    extern __shared__ __align__(16) float lsm[];
    // two buffers of x chunks, [h][token], then two of router_w chunks, [h][expert]
    auto xs = [&](int buf) { return lsm + buf * (HC * TT); };
    auto ws = [&](int buf) { return lsm + 2 * HC * TT + buf * (HC * TE); };

    const int tid = threadIdx.x;
    const int tx = tid % L::NX, ty = tid / L::NX;
    const int t0 = blockIdx.x * TT, e0 = blockIdx.y * TE;
    const bool wvec = (E % 8) == 0;  // router_w rows are 16-byte aligned

    uint4 xr[L::XPT], wrg[L::WPT];
    auto fetch = [&](int h0) {
#pragma unroll
        for (int i = 0; i < L::XPT; ++i) {
            const int v = tid + i * L::NT;
            xr[i] = make_uint4(0, 0, 0, 0);
            if (v < L::XV) {
                const int tt = v % TT, h = h0 + (v / TT) * 8;
                if (t0 + tt < T) xr[i] = *reinterpret_cast<const uint4 *>(x + (size_t)(t0 + tt) * H + h);
            }
        }
#pragma unroll
        for (int i = 0; i < L::WPT; ++i) {
            const int v = tid + i * L::NT;
            wrg[i] = make_uint4(0, 0, 0, 0);
            if (v < L::WV) {
                const int hh = v / (TE / 8), e = e0 + (v % (TE / 8)) * 8;
                const __nv_bfloat16 *src = wr + (size_t)(h0 + hh) * E + e;
                if (wvec && e + 8 <= E) {
                    wrg[i] = *reinterpret_cast<const uint4 *>(src);
                } else {
                    const unsigned short *s16 = reinterpret_cast<const unsigned short *>(src);
                    uint32_t u[4] = {0u, 0u, 0u, 0u};
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        if (e + q < E) u[q / 2] |= static_cast<uint32_t>(s16[q]) << (16 * (q & 1));
                    wrg[i] = make_uint4(u[0], u[1], u[2], u[3]);
                }
            }
        }
    };
    auto stash = [&](int buf) {
#pragma unroll
        for (int i = 0; i < L::XPT; ++i) {
            const int v = tid + i * L::NT;
            if (v < L::XV) {
                const int tt = v % TT, hq = (v / TT) * 8;
                float f[8];
                bf16x8_to_f32(xr[i], f);
#pragma unroll
                for (int q = 0; q < 8; ++q) xs(buf)[(hq + q) * TT + tt] = f[q];
            }
        }
#pragma unroll
        for (int i = 0; i < L::WPT; ++i) {
            const int v = tid + i * L::NT;
            if (v < L::WV) {
                const int hh = v / (TE / 8), e8 = (v % (TE / 8)) * 8;
                float f[8];
                bf16x8_to_f32(wrg[i], f);
                float4 *dst = reinterpret_cast<float4 *>(ws(buf) + hh * TE + e8);
                dst[0] = make_float4(f[0], f[1], f[2], f[3]);
                dst[1] = make_float4(f[4], f[5], f[6], f[7]);
            }
        }
    };

    float acc[RT][RE];
#pragma unroll
    for (int r = 0; r < RT; ++r)
#pragma unroll
        for (int c = 0; c < RE; ++c) acc[r][c] = 0.0f;

    const int nchunks = H / HC;
    fetch(0);
    stash(0);
    __syncthreads();
    for (int ch = 0; ch < nchunks; ++ch) {
        const int buf = ch & 1;
        if (ch + 1 < nchunks) fetch((ch + 1) * HC);
        const float *xb = xs(buf);
        const float *wb = ws(buf);
        // h ascending inside the chunk, chunks ascending: each chain runs h = 0..H-1 in order
#pragma unroll 4
        for (int hh = 0; hh < HC; ++hh) {
            float a[RT], b[RE];
            if constexpr (RT % 4 == 0) {
#pragma unroll
                for (int r = 0; r < RT; r += 4) {
                    const float4 v = *reinterpret_cast<const float4 *>(xb + hh * TT + ty * RT + r);
                    a[r] = v.x; a[r + 1] = v.y; a[r + 2] = v.z; a[r + 3] = v.w;
                }
            } else {
#pragma unroll
                for (int r = 0; r < RT; ++r) a[r] = xb[hh * TT + ty * RT + r];
            }
            if constexpr (RE % 4 == 0) {
#pragma unroll
                for (int c = 0; c < RE; c += 4) {
                    const float4 v = *reinterpret_cast<const float4 *>(wb + hh * TE + tx * RE + c);
                    b[c] = v.x; b[c + 1] = v.y; b[c + 2] = v.z; b[c + 3] = v.w;
                }
            } else {
#pragma unroll
                for (int c = 0; c < RE; ++c) b[c] = wb[hh * TE + tx * RE + c];
            }
#pragma unroll
            for (int r = 0; r < RT; ++r)
#pragma unroll
                for (int c = 0; c < RE; ++c) acc[r][c] = fmaf(a[r], b[c], acc[r][c]);
        }
        if (ch + 1 < nchunks) stash(buf ^ 1);
        __syncthreads();
    }
#pragma unroll
    for (int r = 0; r < RT; ++r) {
        const int t = t0 + ty * RT + r;
#pragma unroll
        for (int c = 0; c < RE; ++c) {
            const int e = e0 + tx * RE + c;
            if (t < T && e < E) {
                float v = acc[r][c];
                if (bias) v = __fadd_rn(v, bias[e]);
                logits[(size_t)t * E + e] = v;
            }
        }
    }
}

template <int TT, int TE, int RT, int RE, int HC>
cudaError_t launch_logits(const __nv_bfloat16 *x, const __nv_bfloat16 *wr, const float *bias, int T, int H,
                          int E, float *logits, cudaStream_t st)
{
    using L = LogitsTile<TT, TE, RT, RE, HC>;
    const size_t smem = (size_t)L::SMEM_FLOATS * sizeof(float);
    auto kern = route_logits_kernel<TT, TE, RT, RE, HC>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    dim3 grid((T + TT - 1) / TT, (E + TE - 1) / TE);
    return launch_pdl(kern, grid, dim3(L::NT), smem, st, x, wr, bias, T, H, E, logits);
}

// Small batches (T <= 32): one chain per thread, TP tokens x TE experts per CTA.
// The chain is latency-bound (H dependent FMAs), so the kernel only has to keep
// its operands arriving and the chain's issue slots free: chunks of HC h-values
// stream into an S-stage shared memory ring with cp.async (16 stages of 128 values
// request the whole H = 2048 slice at once); a thread takes eight x values in one
// 16-byte shared load and feeds them, with its expert's eight weights, to the
// mixed-precision chain step (bf16 operands, fp32 accumulator), one instruction
// per step.
template <int TP, int TE, int HC, int S>
struct SmallTile {
    static constexpr int NT = TP * TE;
    static constexpr int XROW = HC * 2 + 16;            // bytes per token row (padded)
    static constexpr int XBYTES = TP * XROW;
    static constexpr int WBYTES = HC * TE * 2;
    static constexpr int STAGE = XBYTES + WBYTES;
    static constexpr int SMEM = S * STAGE;
};

template <int TP, int TE, int HC, int S>
__global__ void __launch_bounds__(TP * TE)
route_logits_small_kernel(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ wr,
                          const float *__restrict__ bias, int T, int H, int E, float *__restrict__ logits)
{
    pdl_wait();
    pdl_trigger();
    using L = SmallTile<TP, TE, HC, S>;
    extern __shared__ __align__(16) uint8_t ssm[];
    const int tid = threadIdx.x;
    const int tt = tid / TE, ee = tid % TE;
    const int e0 = blockIdx.x * TE;
    const int nchunks = H / HC;

    auto issue = [&](int ch) {
        if (ch < nchunks) {
            uint8_t *st = ssm + (ch % S) * L::STAGE;
            const int h0 = ch * HC;
            for (int v = tid; v < TP * (HC / 8); v += L::NT) {  // x: TP rows of HC values
                const int r = v / (HC / 8), c8 = (v % (HC / 8)) * 8;
                if (r < T) cp_async16(st + r * L::XROW + c8 * 2, x + (size_t)r * H + h0 + c8);
            }
            for (int v = tid; v < HC * (TE / 8); v += L::NT) {  // router_w: HC rows of TE experts
                const int hh = v / (TE / 8), c8 = (v % (TE / 8)) * 8;
                if (e0 + c8 < E) cp_async16(st + L::XBYTES + (hh * TE + c8) * 2, wr + (size_t)(h0 + hh) * E + e0 + c8);
            }
        }
        cp_async_commit();  // one group per chunk slot, empty past the end
    };

    float acc = 0.0f;
#pragma unroll
    for (int s = 0; s < S - 1; ++s) issue(s);
    for (int ch = 0; ch < nchunks; ++ch) {
        cp_async_wait<S - 2>();
        __syncthreads();  // chunk ch visible to all; stage (ch-1)%S free
        issue(ch + S - 1);
        const uint8_t *st = ssm + (ch % S) * L::STAGE;
        const uint4 *xv = reinterpret_cast<const uint4 *>(st + tt * L::XROW);
        const uint16_t *wc = reinterpret_cast<const uint16_t *>(st + L::XBYTES) + ee;
#pragma unroll 4
        for (int h8 = 0; h8 < HC / 8; ++h8) {
            const uint4 xq = xv[h8];
            uint16_t w[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) w[j] = wc[(h8 * 8 + j) * TE];
            acc = chain_step2(xq.x, w[0], w[1], acc);
            acc = chain_step2(xq.y, w[2], w[3], acc);
            acc = chain_step2(xq.z, w[4], w[5], acc);
            acc = chain_step2(xq.w, w[6], w[7], acc);
        }
    }
    cp_async_wait<0>();
    const int e = e0 + ee;
    if (tt < T && e < E) {
        float v = acc;
        if (bias) v = __fadd_rn(v, bias[e]);
        logits[(size_t)tt * E + e] = v;
    }
}

template <int TP, int TE, int HC, int S>
cudaError_t launch_logits_small(const __nv_bfloat16 *x, const __nv_bfloat16 *wr, const float *bias, int T, int H,
                                int E, float *logits, cudaStream_t st)
{
    using L = SmallTile<TP, TE, HC, S>;
    auto kern = route_logits_small_kernel<TP, TE, HC, S>;
    if (L::SMEM > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
        if (e != cudaSuccess) return e;
    }
    return launch_pdl(kern, dim3((E + TE - 1) / TE), dim3(L::NT), L::SMEM, st, x, wr, bias, T, H, E, logits);
}

// Small batches, whole rows resident: the same chains as route_logits_small_kernel
// with the operands brought in by the TMA engine instead of per-thread copies.  x's
// TP rows arrive as untiled bulk copies (one per row, on one barrier); router_w's
// 8-expert column slice arrives as 256 x 8 tiles of a tensor map (one barrier per
// 256 values of h), so the chains start as soon as the first tile lands and no
// thread spends issue slots on staging.  A CTA takes TP = 8 tokens (blockIdx.y) of
// the 8 experts: every step reads a weight and an eighth of an x vector from
// shared memory, so few warps per SM keep the loads under the fma latency.  Needs
// E % 8 == 0, H % 256 == 0 and TP * (2H + 16) + 16H bytes of shared memory.
constexpr int kLogitsChunk = 256;

__host__ __device__ inline size_t logits_tma_smem(int TP, int H)
{
    return 256 + (size_t)TP * (2 * H + 16) + 128 + (size_t)16 * H;
}

template <int TP>
__global__ void __launch_bounds__(TP * 8) route_logits_tma_kernel(const __grid_constant__ CUtensorMap tm_w,
                                                                  const __nv_bfloat16 *__restrict__ x,
                                                                  const float *__restrict__ bias, int T, int H,
                                                                  int E, float *__restrict__ logits,
                                                                  int32_t *__restrict__ status, int clear_status)
{
    extern __shared__ __align__(128) uint8_t tsm_l[];
    constexpr int TE = 8;
    const int nch = H / kLogitsChunk;
    const int pitch = 2 * H + 16;
    uint64_t *bars = reinterpret_cast<uint64_t *>(tsm_l);  // [0]: x rows, [1 + c]: router_w chunk c
    uint8_t *xs = tsm_l + 256;
    uint8_t *wsm = tsm_l + (256 + (size_t)TP * pitch + 127) / 128 * 128;
    const int tid = threadIdx.x, tt = tid / TE, ee = tid % TE;
    const int e0 = blockIdx.x * TE;
    const int t0 = blockIdx.y * TP;
    const int rows = min(TP, T - t0);
    if (tid == 0) {
        for (int i = 0; i <= nch; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
    }
    __syncthreads();
    pdl_wait();
    pdl_trigger();
    if (clear_status && blockIdx.x == 0 && blockIdx.y == 0 && tid == 0) *status = 0;  // first kernel of a forward
    if (tid < 32) {
        if (tid == 0) {
            mbar_arrive_expect_tx(&bars[0], (uint32_t)(rows * H * 2));
            for (int c = 0; c < nch; ++c) {
                mbar_arrive_expect_tx(&bars[1 + c], kLogitsChunk * TE * 2);
                tma_load_2d(wsm + (size_t)c * kLogitsChunk * TE * 2, &tm_w, &bars[1 + c], e0, c * kLogitsChunk);
            }
        }
        __syncwarp();
        for (int r = tid; r < rows; r += 32)
            bulk_load(xs + (size_t)r * pitch, x + (size_t)(t0 + r) * H, H * 2, &bars[0]);
    }
    bool ok = mbar_wait(&bars[0], 0);
    float acc = 0.0f;
    const uint4 *xv = reinterpret_cast<const uint4 *>(xs + (size_t)tt * pitch);
    for (int c = 0; c < nch && ok; ++c) {
        ok = mbar_wait(&bars[1 + c], 0);
        const uint16_t *wc = reinterpret_cast<const uint16_t *>(wsm + (size_t)c * kLogitsChunk * TE * 2) + ee;
        const uint4 *xc = xv + c * (kLogitsChunk / 8);
#pragma unroll
        for (int h8 = 0; h8 < kLogitsChunk / 8; ++h8) {
            const uint4 xq = xc[h8];
            acc = chain_step2(xq.x, wc[(h8 * 8 + 0) * TE], wc[(h8 * 8 + 1) * TE], acc);
            acc = chain_step2(xq.y, wc[(h8 * 8 + 2) * TE], wc[(h8 * 8 + 3) * TE], acc);
            acc = chain_step2(xq.z, wc[(h8 * 8 + 4) * TE], wc[(h8 * 8 + 5) * TE], acc);
            acc = chain_step2(xq.w, wc[(h8 * 8 + 6) * TE], wc[(h8 * 8 + 7) * TE], acc);
        }
    }
    if (!ok) {
        atomicCAS(status, 0, MOE_ERR_TIMEOUT);
        return;
    }
    const int e = e0 + ee;
    if (tt < rows && e < E) {
        float v = acc;
        if (bias) v = __fadd_rn(v, bias[e]);
        logits[(size_t)(t0 + tt) * E + e] = v;
    }
}

// Launches the TMA-fed kernel when the shape allows it (returns false otherwise).
template <int TP>
bool try_launch_logits_tma(const __nv_bfloat16 *x, const __nv_bfloat16 *wr, const float *bias, int T, int H, int E,
                           float *logits, int32_t *status, int clear_status, cudaStream_t st, cudaError_t *err)
{
    const size_t smem = logits_tma_smem(TP, H);
    if (E % 8 || H % kLogitsChunk || H / kLogitsChunk > 31 || smem > 227 * 1024) return false;
    CUtensorMap tm;
    if (!encode_plain_2d_bf16(&tm, wr, H, E, 8, kLogitsChunk)) return false;
    auto kern = route_logits_tma_kernel<TP>;
    *err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (*err != cudaSuccess) return true;
    *err = launch_pdl(kern, dim3(E / 8, (T + TP - 1) / TP), dim3(TP * 8), smem, st, tm, x, bias, T, H, E, logits,
                      status, clear_status);
    return true;
}

// The small-batch logits: TMA-fed when the rows fit in shared memory, else the
// cp.async ring.  With clear_status the status word is zeroed first (by the TMA
// kernel, or by a memset ahead of the cp.async one).
cudaError_t launch_logits_small_any(const __nv_bfloat16 *x, const __nv_bfloat16 *wr, const float *bias, int T,
                                    int H, int E, float *logits, int32_t *status, cudaStream_t st,
                                    bool clear_status = false)
{
    cudaError_t err = cudaSuccess;
    if (try_launch_logits_tma<8>(x, wr, bias, T, H, E, logits, status, clear_status, st, &err)) return err;
    if (clear_status && (err = cudaMemsetAsync(status, 0, sizeof(int32_t), st)) != cudaSuccess) return err;
    return T <= 16 ? launch_logits_small<16, 8, 128, 16>(x, wr, bias, T, H, E, logits, st)
                   : launch_logits_small<32, 8, 128, 16>(x, wr, bias, T, H, E, logits, st);
}

// Loads one token's logits into the warp_topk layout (expert lane + 32 i).
template <int MAXV>
__device__ __forceinline__ void load_logit_row(const float *__restrict__ lrow, int E, uint32_t (&key)[MAXV],
                                               float (&val)[MAXV])
{
    const int lane = threadIdx.x % 32;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
        const int e = lane + 32 * i;
        val[i] = e < E ? lrow[e] : 0.0f;
        key[i] = e < E ? order_key(val[i]) : 0u;
    }
}

// Softmax over the k chosen logits v[0..k-1] (v[0] the largest), fp32 with the
// maximum subtracted; lanes write gates j = lane, lane + 32, ...
__device__ __forceinline__ void gates_softmax(const float *v, int k, float *__restrict__ gate_out)
{
    const int lane = threadIdx.x % 32;
    const float m = v[0];
    float s = 0.0f;
    for (int j = lane; j < k; j += 32) s += expf(v[j] - m);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    for (int j = lane; j < k; j += 32) gate_out[j] = expf(v[j] - m) / s;
}

template <int MAXV>
__global__ void route_topk_kernel(const float *__restrict__ logits, int T, int E, int k,
                                  int32_t *__restrict__ idx, float *__restrict__ gate)
{
    pdl_wait();
    pdl_trigger();
    extern __shared__ __align__(16) uint8_t tksm[];  // [warps][k] experts, then [warps][k] values
    const int warp = threadIdx.x / 32, nw = blockDim.x / 32, lane = threadIdx.x % 32;
    const int t = blockIdx.x * nw + warp;
    if (t >= T) return;
    int *se = reinterpret_cast<int *>(tksm) + (size_t)warp * k;
    float *sv = reinterpret_cast<float *>(tksm) + (size_t)nw * k + (size_t)warp * k;
    uint32_t key[MAXV];
    float val[MAXV];
    load_logit_row<MAXV>(logits + (size_t)t * E, E, key, val);
    warp_topk<MAXV>(key, val, k, se, sv);
    for (int j = lane; j < k; j += 32) idx[(size_t)t * k + j] = se[j];
    gates_softmax(sv, k, gate + (size_t)t * k);
}

template <int MAXV>
cudaError_t launch_topk(const float *logits, int T, int E, int k, int32_t *idx, float *gate,
                        cudaStream_t st)
{
    constexpr int warps = 8;
    const size_t smem = (size_t)warps * k * 8;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(route_topk_kernel<MAXV>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    return launch_pdl(route_topk_kernel<MAXV>, dim3((T + warps - 1) / warps), dim3(warps * 32), smem, st, logits, T,
                      E, k, idx, gate);
}

// ------------------------------------------------------------------------
// Small batches inside the forward: route_logits_small_kernel, then one CTA that
// does top-k + softmax per token (a warp each) and the stable grouping by expert
// of the A = T*k assignments -- the same results as route_topk_kernel and the
// three permute kernels of permute.cu.
//
// Grouping: chunk c holds the flat entries 32c..32c+31 and belongs to warp c % nw.
//  1. each warp ranks its chunk's entries among equal experts (__match_any_sync)
//     and records tbl[c][e], the chunk's count of expert e;
//  2. a thread per expert turns tbl[.][e] into the exclusive prefix over chunks
//     (chunks ascending) and its total;
//  3. a block-wide scan of the totals over experts (a thread per run of experts):
//     offsets, the tile list {expert, row_start, rows} and the number of tiles;
//  4. entry f of chunk c on expert e lands at offsets[e] + tbl[c][e] + rank.
// So equal experts keep flat order (a stable counting sort) with six barriers.
struct SmallRouteOut {
    float *logits;
    int32_t *idx;
    float *gate;
    int32_t *offsets, *s2f, *f2s, *tiles, *ntiles;
    int32_t *counters;
    int ncounters;
    int32_t *ccnt;   // the fused combine's arrival counts, zeroed here
    int nccnt;
    int32_t *status;
};

constexpr int kSmallTblMax = 16384;  // chunk x expert entries of the grouping table

__host__ __device__ inline size_t small_topk_permute_smem(int T, int E, int k, int warps)
{
    const int A = T * k, nch = (A + 31) / 32;
    return ((size_t)A + 2 * (size_t)warps * k + E + (size_t)nch * E) * 4;
}

template <int MAXV>
__global__ void __launch_bounds__(1024) topk_permute_small_kernel(int T, int E, int k, SmallRouteOut o)
{
    pdl_wait();
    pdl_trigger();
    extern __shared__ __align__(16) uint8_t tsm[];
    const int tid = threadIdx.x, NT = blockDim.x, lane = tid % 32, warp = tid / 32, nw = NT / 32;
    const int A = T * k, nch = (A + 31) / 32;
    int *sidx = reinterpret_cast<int *>(tsm);           // [A] chosen experts, flat order
    int *se = sidx + A;                                  // [nw][k]
    float *sv = reinterpret_cast<float *>(se + nw * k);  // [nw][k]
    int *base = reinterpret_cast<int *>(sv + nw * k);    // [E] first sorted row of each expert
    int *tbl = base + E;                                 // [nch][E]

    for (int i = tid; i < nch * E; i += NT) tbl[i] = 0;
    for (int t = warp; t < T; t += nw) {
        uint32_t key[MAXV];
        float val[MAXV];
        load_logit_row<MAXV>(o.logits + (size_t)t * E, E, key, val);
        int *e_out = se + warp * k;
        float *v_out = sv + warp * k;
        warp_topk<MAXV>(key, val, k, e_out, v_out);
        for (int j = lane; j < k; j += 32) {
            sidx[t * k + j] = e_out[j];
            o.idx[(size_t)t * k + j] = e_out[j];
        }
        gates_softmax(v_out, k, o.gate + (size_t)t * k);
        __syncwarp();
    }
    __syncthreads();
    // 1. per-chunk counts
    for (int c = warp; c < nch; c += nw) {
        const int f = c * 32 + lane;
        const int e = f < A ? sidx[f] : -1;
        const bool valid = e >= 0 && e < E;
        if (f < A && !valid) atomicCAS(o.status, 0, MOE_ERR_BAD_INDEX);
        const unsigned peers = __match_any_sync(0xffffffffu, valid ? e : -1);
        if (valid && (peers & ((1u << lane) - 1u)) == 0u) tbl[c * E + e] = __popc(peers);
    }
    __syncthreads();
    // 2. exclusive prefix over chunks, per expert
    for (int e = tid; e < E; e += NT) {
        int run = 0;
        for (int c = 0; c < nch; ++c) {
            const int v = tbl[c * E + e];
            tbl[c * E + e] = run;
            run += v;
        }
        base[e] = run;
    }
    __syncthreads();
    // 3. offsets and tile list: thread i takes experts i*per .. i*per + per - 1, and a
    // block-wide exclusive scan of (rows, tiles) in expert order places them (the
    // warps' totals in se[], free after the top-k)
    {
        const int per = (E + NT - 1) / NT;
        const int lo = min(E, tid * per), hi = min(E, lo + per);
        int rows = 0, tls = 0;
        for (int e = lo; e < hi; ++e) {
            rows += base[e];
            tls += (base[e] + kTileRows - 1) / kTileRows;
        }
        int rinc = rows, tinc = tls;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int r = __shfl_up_sync(0xffffffffu, rinc, off);
            const int q = __shfl_up_sync(0xffffffffu, tinc, off);
            if (lane >= off) {
                rinc += r;
                tinc += q;
            }
        }
        int *wrow = se, *wtil = se + nw;  // 2 nw <= 2 nw k entries
        if (lane == 31) {
            wrow[warp] = rinc;
            wtil[warp] = tinc;
        }
        __syncthreads();
        if (warp == 0) {
            int r = lane < nw ? wrow[lane] : 0, q = lane < nw ? wtil[lane] : 0;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int r2 = __shfl_up_sync(0xffffffffu, r, off);
                const int q2 = __shfl_up_sync(0xffffffffu, q, off);
                if (lane >= off) {
                    r += r2;
                    q += q2;
                }
            }
            if (lane < nw) {  // inclusive prefix over the warps
                wrow[lane] = r;
                wtil[lane] = q;
            }
        }
        __syncthreads();
        const int rbase = warp > 0 ? wrow[warp - 1] : 0, tbase = warp > 0 ? wtil[warp - 1] : 0;
        int off = rbase + rinc - rows, toff = tbase + tinc - tls;
        for (int e = lo; e < hi; ++e) {
            const int c = base[e];
            o.offsets[e] = off;
            for (int m = 0; m * kTileRows < c; ++m) {
                int32_t *tl = o.tiles + 3 * (size_t)(toff + m);
                tl[0] = e;
                tl[1] = off + m * kTileRows;
                tl[2] = min(kTileRows, c - m * kTileRows);
            }
            toff += (c + kTileRows - 1) / kTileRows;
            base[e] = off;
            off += c;
        }
        if (tid == NT - 1) {
            o.offsets[E] = wrow[nw - 1];
            *o.ntiles = wtil[nw - 1];
        }
    }
    __syncthreads();
    // 4. scatter
    for (int c = warp; c < nch; c += nw) {
        const int f = c * 32 + lane;
        const int e = f < A ? sidx[f] : -1;
        const bool valid = e >= 0 && e < E;
        const unsigned peers = __match_any_sync(0xffffffffu, valid ? e : -1);
        if (valid) {
            const int pos = base[e] + tbl[c * E + e] + __popc(peers & ((1u << lane) - 1u));
            o.s2f[pos] = f;
            o.f2s[f] = pos;
        }
    }
    if (tid < o.ncounters) o.counters[tid] = 0;
    for (int i = tid; i < o.nccnt; i += NT) o.ccnt[i] = 0;
}

}  // namespace

bool small_route_permute_ok(const moe_dims_t &d)
{
    const long A = (long)d.T * d.top_k;
    return d.T <= 32 && d.E % 8 == 0 && d.H % 128 == 0 && A <= 4096 && ((A + 31) / 32) * d.E <= kSmallTblMax;
}

cudaError_t launch_route_permute_small(const moe_dims_t &d, const __nv_bfloat16 *x, const __nv_bfloat16 *wr,
                                       const float *bias, float *logits, int32_t *idx, float *gate,
                                       int32_t *offsets, int32_t *s2f, int32_t *f2s, int32_t *tiles,
                                       int32_t *ntiles, WsHeader *hdr, int32_t *ccnt, int nccnt, cudaStream_t st)
{
    SmallRouteOut o{logits, idx, gate, offsets, s2f, f2s, tiles, ntiles, hdr->counter, 7, ccnt, nccnt, &hdr->status};
    cudaError_t e = launch_logits_small_any(x, wr, bias, d.T, d.H, d.E, logits, &hdr->status, st, true);
    if (e != cudaSuccess) return e;
    const int warps = d.T < 4 ? 4 : d.T;
    const size_t smem = small_topk_permute_smem(d.T, d.E, d.top_k, warps);
    const int vpl = (d.E + 31) / 32;
    auto launch = [&](auto kern) {
        if (smem > 48 * 1024) {
            cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (r != cudaSuccess) return r;
        }
        return launch_pdl(kern, dim3(1), dim3(warps * 32), smem, st, d.T, d.E, d.top_k, o);
    };
    if (vpl <= 1) return launch(topk_permute_small_kernel<1>);
    if (vpl <= 2) return launch(topk_permute_small_kernel<2>);
    if (vpl <= 4) return launch(topk_permute_small_kernel<4>);
    if (vpl <= 8) return launch(topk_permute_small_kernel<8>);
    if (vpl <= 16) return launch(topk_permute_small_kernel<16>);
    return launch(topk_permute_small_kernel<32>);
}

cudaError_t launch_route(const moe_dims_t &d, const __nv_bfloat16 *x, const __nv_bfloat16 *wr,
                         const float *bias, float *logits, int32_t *idx, float *gate,
                         const RouterScratch &rs, WsHeader *hdr, cudaStream_t st)
{
    const int T = d.T, H = d.H, E = d.E, k = d.top_k;
    if (T > 32) return launch_route_certified(d, x, wr, bias, logits, idx, gate, rs, hdr, st);
    cudaError_t e;
    if (E % 8 == 0 && H % 128 == 0)
        e = launch_logits_small_any(x, wr, bias, T, H, E, logits, &hdr->status, st);
    else
        e = launch_logits<16, 16, 1, 1, 64>(x, wr, bias, T, H, E, logits, st);
    if (e != cudaSuccess) return e;
    const int vpl = (E + 31) / 32;
    if (vpl <= 1) return launch_topk<1>(logits, T, E, k, idx, gate, st);
    if (vpl <= 2) return launch_topk<2>(logits, T, E, k, idx, gate, st);
    if (vpl <= 4) return launch_topk<4>(logits, T, E, k, idx, gate, st);
    if (vpl <= 8) return launch_topk<8>(logits, T, E, k, idx, gate, st);
    if (vpl <= 16) return launch_topk<16>(logits, T, E, k, idx, gate, st);
    return launch_topk<32>(logits, T, E, k, idx, gate, st);
}

}  // namespace moe
