// route.cu -- router logits and softmax top-k gating.
//
// The router picks, for every token, the top-k experts by router logit and
// weights their outputs by a softmax over the chosen k (vLLM fused-MoE page,
// section 02; the Weave review, section 1.1, describes the same top-k router).
//
// Logit contract: logit[t,e] is the fp32 result of the fused-multiply-add chain
// over h = 0..H-1 in ascending order starting from 0.0f, followed by one fp32
// addition of bias[e].  Every (t,e) chain is evaluated by one thread in exactly
// that order, so the logits -- and the integer routing decision taken on them --
// are reproducible bit for bit.
//
// Kernel 1 (route_logits): a CUDA-core tile of TT tokens x TE experts per CTA,
//   operands staged in double-buffered shared memory as fp32 (bf16 -> fp32 is
//   exact), the next chunk prefetched into registers, each thread owning RT x RE
//   independent chains.
// Kernel 2 (route_topk): one warp per token; k rounds of a warp arg-max with the
//   (larger logit, then lower index) order, then the softmax over the k chosen
//   logits with the maximum subtracted.
#include <cfloat>
#include <climits>

#include "moe_internal.h"

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

// Small batches (T <= 32): one chain per thread, TP tokens x TE experts per CTA.
// The chain is latency-bound (H dependent FMAs), so the kernel only has to keep
// its operands arriving: chunks of HC h-values stream into an S-stage shared
// memory ring with cp.async (bf16, converted at use), S-1 chunks in flight --
// with 16 stages of 128 values the whole H = 2048 slice is requested at once.
template <int TP, int TE, int HC, int S>
struct SmallTile {
    static constexpr int NT = TP * TE;
    static constexpr int XROW = HC * 2 + 16;            // bytes per token row (padded)
    static constexpr int XBYTES = TP * XROW;
    static constexpr int WBYTES = HC * TE * 2;
    static constexpr int STAGE = XBYTES + WBYTES;
    static constexpr int SMEM = S * STAGE;
};

__device__ __forceinline__ void cp_async16(void *dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int TP, int TE, int HC, int S>
__global__ void __launch_bounds__(TP * TE)
route_logits_small_kernel(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ wr,
                          const float *__restrict__ bias, int T, int H, int E, float *__restrict__ logits)
{
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
        __syncthreads();             // chunk ch visible to all; stage (ch-1)%S free
        issue(ch + S - 1);
        const uint8_t *st = ssm + (ch % S) * L::STAGE;
        const __nv_bfloat16 *xr = reinterpret_cast<const __nv_bfloat16 *>(st + tt * L::XROW);
        const __nv_bfloat16 *wc = reinterpret_cast<const __nv_bfloat16 *>(st + L::XBYTES) + ee;
#pragma unroll 8
        for (int hh = 0; hh < HC; ++hh)
            acc = fmaf(__bfloat162float(xr[hh]), __bfloat162float(wc[hh * TE]), acc);
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
    kern<<<(E + TE - 1) / TE, L::NT, L::SMEM, st>>>(x, wr, bias, T, H, E, logits);
    return cudaGetLastError();
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
    kern<<<grid, L::NT, smem, st>>>(x, wr, bias, T, H, E, logits);
    return cudaGetLastError();
}

// (v1, e1) ranks before (v2, e2): larger logit first, equal logits -> lower index.
__device__ __forceinline__ bool ranks_before(float v1, int e1, float v2, int e2)
{
    if (e2 == INT_MAX) return e1 != INT_MAX;
    if (e1 == INT_MAX) return false;
    return v1 > v2 || (v1 == v2 && e1 < e2);
}

// One warp: top-k of one token's E logits (larger logit first, equal logits ->
// lower index) and the softmax over the chosen k.  `sv` is k floats of scratch.
template <int MAXV>
__device__ __forceinline__ void topk_softmax_warp(const float *__restrict__ lrow, int E, int k,
                                                  int32_t *__restrict__ idx_out, float *__restrict__ gate_out,
                                                  float *sv)
{
    const int lane = threadIdx.x % 32;
    float v[MAXV];
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
        const int e = lane + 32 * i;
        v[i] = e < E ? lrow[e] : 0.0f;
    }
    uint32_t taken = 0;
    for (int j = 0; j < k; ++j) {
        float bv = 0.0f;
        int be = INT_MAX;
#pragma unroll
        for (int i = 0; i < MAXV; ++i) {
            const int e = lane + 32 * i;
            if (e < E && !((taken >> i) & 1u) && ranks_before(v[i], e, bv, be)) {
                bv = v[i];
                be = e;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oe = __shfl_xor_sync(0xffffffffu, be, off);
            if (ranks_before(ov, oe, bv, be)) {
                bv = ov;
                be = oe;
            }
        }
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        if (lane == 0) {
            idx_out[j] = be;
            sv[j] = bv;
        }
    }
    __syncwarp();
    const float m = sv[0];  // the first choice holds the largest logit
    float s = 0.0f;
    for (int j = lane; j < k; j += 32) s += expf(sv[j] - m);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    for (int j = lane; j < k; j += 32) gate_out[j] = expf(sv[j] - m) / s;
    __syncwarp();
}

template <int MAXV>
__global__ void route_topk_kernel(const float *__restrict__ logits, int T, int E, int k,
                                  int32_t *__restrict__ idx, float *__restrict__ gate)
{
    extern __shared__ float sel[];  // [warps][k] chosen logits
    const int warp = threadIdx.x / 32;
    const int t = blockIdx.x * (blockDim.x / 32) + warp;
    if (t >= T) return;
    topk_softmax_warp<MAXV>(logits + (size_t)t * E, E, k, idx + (size_t)t * k, gate + (size_t)t * k,
                            sel + (size_t)warp * k);
}

template <int MAXV>
cudaError_t launch_topk(const float *logits, int T, int E, int k, int32_t *idx, float *gate,
                        cudaStream_t st)
{
    constexpr int warps = 8;
    const size_t smem = (size_t)warps * k * sizeof(float);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(route_topk_kernel<MAXV>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    route_topk_kernel<MAXV><<<(T + warps - 1) / warps, warps * 32, smem, st>>>(logits, T, E, k, idx,
                                                                              gate);
    return cudaGetLastError();
}

// ------------------------------------------------------------------------
// Small batches, router + permute in two launches.  route_logits_pipe_kernel is
// route_logits_small_kernel with the chain fed from registers: eight x values
// arrive in one 16-byte shared load and the next eight (and their weights) are
// loaded while the current eight feed the FMA chain.  topk_permute_small_kernel
// then runs one CTA: top-k and softmax per token (a warp each) and the stable
// grouping by expert of the T*k assignments -- the same results as
// route_topk_kernel and the three permute kernels.
struct SmallRouteOut {
    float *logits;
    int32_t *idx;
    float *gate;
    int32_t *offsets, *s2f, *f2s, *tiles, *ntiles;
    int32_t *counters;
    int ncounters;
    int32_t *status;
};

// Exclusive scan of one value per thread over the CTA (blockDim <= 1024).
__device__ int cta_exclusive_scan(int v, int *wtot, int &total)
{
    const int lane = threadIdx.x % 32, warp = threadIdx.x / 32, nw = blockDim.x / 32;
    int inc = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, inc, off);
        if (lane >= off) inc += o;
    }
    if (lane == 31) wtot[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        const int w = lane < nw ? wtot[lane] : 0;
        int wi = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, wi, off);
            if (lane >= off) wi += o;
        }
        if (lane < nw) wtot[lane] = wi - w;
        if (lane == 31) wtot[32] = wi;
    }
    __syncthreads();
    const int res = wtot[warp] + inc - v;
    total = wtot[32];
    __syncthreads();
    return res;
}

// Stable counting sort of A flat assignments by expert inside one CTA (A small).
__device__ void permute_in_cta(const int32_t *__restrict__ idx, int A, int E, const SmallRouteOut &o, int *sm)
{
    const int NT = blockDim.x, tid = threadIdx.x, lane = tid % 32, warp = tid / 32, nw = NT / 32;
    int *cursor = sm;             // [E]
    int *wtot = sm + E;           // [33]
    for (int e = tid; e < E; e += NT) cursor[e] = 0;
    __syncthreads();
    for (int f = tid; f < A; f += NT) {
        const int e = idx[f];
        if (e >= 0 && e < E)
            atomicAdd(&cursor[e], 1);
        else
            atomicCAS(o.status, 0, MOE_ERR_BAD_INDEX);
    }
    __syncthreads();
    // each thread owns a contiguous run of experts for the two scans
    const int per = (E + NT - 1) / NT;
    const int e_lo = min(E, tid * per), e_hi = min(E, e_lo + per);
    int rows = 0, tls = 0;
    for (int e = e_lo; e < e_hi; ++e) {
        rows += cursor[e];
        tls += (cursor[e] + kTileRows - 1) / kTileRows;
    }
    int total_rows = 0, total_tiles = 0;
    int off = cta_exclusive_scan(rows, wtot, total_rows);
    int toff = cta_exclusive_scan(tls, wtot, total_tiles);
    for (int e = e_lo; e < e_hi; ++e) {
        const int c = cursor[e];
        o.offsets[e] = off;
        for (int m = 0; m * kTileRows < c; ++m) {
            int32_t *tl = o.tiles + 3 * (size_t)(toff + m);
            tl[0] = e;
            tl[1] = off + m * kTileRows;
            tl[2] = min(kTileRows, c - m * kTileRows);
        }
        toff += (c + kTileRows - 1) / kTileRows;
        cursor[e] = off;  // becomes the next free sorted row of expert e
        off += c;
    }
    if (tid == 0) {
        o.offsets[E] = total_rows;
        *o.ntiles = total_tiles;
    }
    __syncthreads();
    // chunks in order; inside a chunk, warps in order; inside a warp, lanes by rank
    for (int c0 = 0; c0 < A; c0 += NT) {
        const int f = c0 + tid;
        const int e = f < A ? idx[f] : -1;
        const bool valid = e >= 0 && e < E;
        const unsigned peers = __match_any_sync(0xffffffffu, valid ? e : -1);
        const int rank = __popc(peers & ((1u << lane) - 1u));
        for (int w = 0; w < nw; ++w) {
            if (warp == w && valid) {
                const int pos = cursor[e] + rank;
                o.s2f[pos] = f;
                o.f2s[f] = pos;
            }
            __syncwarp();
            if (warp == w && valid && rank == 0) cursor[e] += __popc(peers);
            __syncthreads();
        }
    }
    if (tid < o.ncounters) o.counters[tid] = 0;
}

template <int TP, int TE, int HC, int S>
__global__ void __launch_bounds__(TP * TE)
route_logits_pipe_kernel(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ wr,
                         const float *__restrict__ bias, int T, int H, int E, float *__restrict__ logits)
{
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
            for (int v = tid; v < TP * (HC / 8); v += L::NT) {
                const int r = v / (HC / 8), c8 = (v % (HC / 8)) * 8;
                if (r < T) cp_async16(st + r * L::XROW + c8 * 2, x + (size_t)r * H + h0 + c8);
            }
            for (int v = tid; v < HC * (TE / 8); v += L::NT) {
                const int hh = v / (TE / 8), c8 = (v % (TE / 8)) * 8;
                if (e0 + c8 < E) cp_async16(st + L::XBYTES + (hh * TE + c8) * 2, wr + (size_t)(h0 + hh) * E + e0 + c8);
            }
        }
        cp_async_commit();
    };

    float acc = 0.0f;
#pragma unroll
    for (int s = 0; s < S - 1; ++s) issue(s);
    for (int ch = 0; ch < nchunks; ++ch) {
        cp_async_wait<S - 2>();
        __syncthreads();
        issue(ch + S - 1);
        const uint8_t *st = ssm + (ch % S) * L::STAGE;
        const uint4 *xv = reinterpret_cast<const uint4 *>(st + tt * L::XROW);
        const unsigned short *wc = reinterpret_cast<const unsigned short *>(st + L::XBYTES) + ee;
        uint4 xq = xv[0];
        unsigned short w[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) w[j] = wc[j * TE];
#pragma unroll
        for (int h8 = 0; h8 < HC / 8; ++h8) {
            uint4 xn = xq;
            unsigned short wn[8];
            if (h8 + 1 < HC / 8) {
                xn = xv[h8 + 1];
#pragma unroll
                for (int j = 0; j < 8; ++j) wn[j] = wc[((h8 + 1) * 8 + j) * TE];
            }
            const uint32_t xw[4] = {xq.x, xq.y, xq.z, xq.w};
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float a = __uint_as_float((j & 1) ? (xw[j / 2] & 0xFFFF0000u) : (xw[j / 2] << 16));
                const float b = __uint_as_float(static_cast<uint32_t>(w[j]) << 16);
                acc = fmaf(a, b, acc);
            }
            xq = xn;
            if (h8 + 1 < HC / 8) {
#pragma unroll
                for (int j = 0; j < 8; ++j) w[j] = wn[j];
            }
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

// Top-k + softmax for every token (one warp per token) and the stable grouping by
// expert of the T*k assignments, in one CTA: small batches only (T <= 32).
template <int MAXV>
__global__ void __launch_bounds__(1024) topk_permute_small_kernel(int T, int E, int k, SmallRouteOut o)
{
    extern __shared__ __align__(16) uint8_t tsm[];
    const int warp = threadIdx.x / 32, nw = blockDim.x / 32;
    float *sv = reinterpret_cast<float *>(tsm);  // [nw][k]
    for (int t = warp; t < T; t += nw)
        topk_softmax_warp<MAXV>(o.logits + (size_t)t * E, E, k, o.idx + (size_t)t * k, o.gate + (size_t)t * k,
                                sv + (size_t)warp * k);
    __syncthreads();
    permute_in_cta(o.idx, T * k, E, o, reinterpret_cast<int *>(tsm) + nw * k);
}


// ------------------------------------------------------------------------
// Large batches: tensor-core logits certified against the fp32 chain.
//
// The router's logit is defined by the fp32 FMA chain; computing all T*E chains
// costs 2*T*H*E CUDA-core flops.  For T > 32 the chain is instead evaluated only
// where it can change the answer:
//  1. Lt = x . Wr on the tensor cores (bf16 in, fp32 accumulate), each 64-wide K
//     block summed out of TMEM in fp32 and K split over a few slices, against Wr
//     transposed to [E, H] once per call.
//  2. Per token, a bound |chain - Lt| <= d_e: the chain's own rounding is at most
//     H u sum_h |x_h w_he| (u = 2^-24, recursive summation with fma), the
//     tensor-core value's at most (64 * 4u + (H/64 + slices) u) times the same sum
//     (each 64-term block accumulated within 4 ulps, then one rounding per block and
//     slice sum); sum_h |x_h w_he| <= |x_t| |w_e| (Cauchy-Schwarz); 1% margin, plus
//     a few ulps of the bias add and of the values themselves.
//  3. tau = the k-th largest lower bound Lt - d.  An expert whose upper bound
//     Lt + d is below tau has k experts strictly above it, so it cannot be chosen.
//     The remaining candidates (k of them plus near-ties) go to a compact list
//     (kernel C1, a warp per token), get the exact chain (C2, a thread per
//     candidate), and top-k + softmax run on those exact values (C3).
//  4. Every candidate's exact value is checked against its bound; a miss records
//     MOE_ERR_ROUTER_BOUND in the status word.
// The chosen experts and gates are therefore those of the chain definition.

__global__ void router_transpose_kernel(const __nv_bfloat16 *__restrict__ wr, int H, int E,
                                        __nv_bfloat16 *__restrict__ wrt)
{
    __shared__ __nv_bfloat16 tile[32][33];
    const int h0 = blockIdx.y * 32, e0 = blockIdx.x * 32;
    const int tx = threadIdx.x % 32, ty = threadIdx.x / 32;  // 32 x 8 threads
    for (int r = ty; r < 32; r += 8) {
        const int h = h0 + r, e = e0 + tx;
        tile[r][tx] = (h < H && e < E) ? wr[(size_t)h * E + e] : __float2bfloat16(0.0f);
    }
    __syncthreads();
    for (int r = ty; r < 32; r += 8) {
        const int e = e0 + r, h = h0 + tx;
        if (e < E && h < H) wrt[(size_t)e * H + h] = tile[tx][r];
    }
}

// Squared norm of each router column (warp per expert, fp32; the bound inflates it).
__global__ void router_colnorm_kernel(const __nv_bfloat16 *__restrict__ wrt, int H, int E, float *__restrict__ wsq)
{
    const int e = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32, lane = threadIdx.x % 32;
    if (e >= E) return;
    float s = 0.0f;
    for (int h = lane * 8; h < H; h += 256) {
        float f[8];
        bf16x8_to_f32(*reinterpret_cast<const uint4 *>(wrt + (size_t)e * H + h), f);
#pragma unroll
        for (int i = 0; i < 8; ++i) s = fmaf(f[i], f[i], s);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) wsq[e] = s;
}

// The exact chain of one (token, expert): fma over h ascending from 0, operands
// streamed from global memory (L1/L2) sixteen 16-byte loads ahead so that the
// loads' latency hides behind the chain.
__device__ __forceinline__ float exact_chain(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ w,
                                             int H)
{
    constexpr int D = 16;  // loads in flight per operand
    const uint4 *w4 = reinterpret_cast<const uint4 *>(w);
    const uint4 *x4 = reinterpret_cast<const uint4 *>(x);
    const int n8 = H / 8;  // H is a multiple of 64
    float acc = 0.0f;
    uint4 wq[D], xq[D];
#pragma unroll
    for (int j = 0; j < D; ++j) {
        wq[j] = j < n8 ? w4[j] : make_uint4(0, 0, 0, 0);
        xq[j] = j < n8 ? x4[j] : make_uint4(0, 0, 0, 0);
    }
    for (int b = 0; b < n8; b += D) {
#pragma unroll
        for (int j = 0; j < D; ++j) {
            if (b + j < n8) {
                const uint4 wv = wq[j], xv = xq[j];
                if (b + j + D < n8) {
                    wq[j] = w4[b + j + D];
                    xq[j] = x4[b + j + D];
                }
                const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w}, xx[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    acc = fmaf(__uint_as_float(xx[i] << 16), __uint_as_float(ww[i] << 16), acc);
                    acc = fmaf(__uint_as_float(xx[i] & 0xFFFF0000u), __uint_as_float(ww[i] & 0xFFFF0000u), acc);
                }
            }
        }
    }
    return acc;
}

struct CertifyArgs {
    const float *lt;        // [ksplit, T, E] partial tensor-core logits; slice 0 later holds exact values
    int ksplit;
    const __nv_bfloat16 *x, *wrt;
    const float *wsq, *bias;
    int T, H, E, k;
    float eps;
    int32_t *ncand;         // [T] candidates per token
    int32_t *cand;          // [T, E] candidate experts, ascending
    RouterCand *list;       // compact list of all candidates
    int32_t *list_len;
    float *ex;              // [T, E] exact chain values (written for candidates only)
    int32_t *idx;
    float *gate;
    int32_t *status;
};

// C1: bounds and candidates, one warp per token.
template <int MAXV>
__global__ void __launch_bounds__(256) router_candidates_kernel(const CertifyArgs a)
{
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int t = blockIdx.x * (blockDim.x / 32) + warp;
    if (t >= a.T) return;
    const int E = a.E, H = a.H;
    // tensor-core logits (sum of the K slices) first, so their loads overlap the norm
    float v[MAXV], d[MAXV];
#pragma unroll
    for (int i = 0; i < MAXV; ++i) v[i] = 0.0f;
    for (int q = 0; q < a.ksplit; ++q) {
        const float *row = a.lt + ((size_t)q * a.T + t) * E;
#pragma unroll
        for (int i = 0; i < MAXV; ++i) {
            const int e = lane + 32 * i;
            if (e < E) v[i] += row[e];
        }
    }
    float ss = 0.0f;
    const uint4 *xr = reinterpret_cast<const uint4 *>(a.x + (size_t)t * H);
#pragma unroll 4
    for (int h8 = lane; h8 < H / 8; h8 += 32) {
        float f[8];
        bf16x8_to_f32(xr[h8], f);
#pragma unroll
        for (int i = 0; i < 8; ++i) ss = fmaf(f[i], f[i], ss);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float xn = sqrtf(ss) * 1.001f;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
        const int e = lane + 32 * i;
        if (e < E) {
            float s = v[i];
            if (a.bias) s += a.bias[e];
            v[i] = s;
            d[i] = a.eps * xn * sqrtf(a.wsq[e]) * 1.001f + fabsf(s) * 4.8e-7f + 1e-30f;
        } else {
            v[i] = -INFINITY;
            d[i] = 0.0f;
        }
    }
    // tau: the k-th largest lower bound v - d
    uint32_t taken = 0;
    float tau = -INFINITY;
    for (int j = 0; j < a.k; ++j) {
        float bv = -INFINITY;
        int be = INT_MAX;
#pragma unroll
        for (int i = 0; i < MAXV; ++i) {
            const int e = lane + 32 * i;
            const float lo = v[i] - d[i];
            if (e < E && !((taken >> i) & 1u) && (be == INT_MAX || lo > bv)) {
                bv = lo;
                be = e;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oe = __shfl_xor_sync(0xffffffffu, be, off);
            if (oe != INT_MAX && (be == INT_MAX || ov > bv || (ov == bv && oe < be))) {
                bv = ov;
                be = oe;
            }
        }
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        tau = bv;
    }
    // candidates (upper bound >= tau), ascending expert index, appended contiguously
    int nc = 0;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
        const int e = lane + 32 * i;
        nc += __popc(__ballot_sync(0xffffffffu, e < E && v[i] + d[i] >= tau));
    }
    int base = 0;
    if (lane == 0) base = atomicAdd(a.list_len, nc);
    base = __shfl_sync(0xffffffffu, base, 0);
    int pos = 0;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
        const int e = lane + 32 * i;
        const bool c = e < E && v[i] + d[i] >= tau;
        const unsigned m = __ballot_sync(0xffffffffu, c);
        if (c) {
            const int p = pos + __popc(m & ((1u << lane) - 1u));
            a.cand[(size_t)t * E + p] = e;
            a.list[base + p] = RouterCand{t, e, v[i], d[i]};
        }
        pos += __popc(m);
    }
    if (lane == 0) a.ncand[t] = nc;
}

// C2: the exact chain of every candidate, one thread each; checked against its bound.
__global__ void __launch_bounds__(128) router_chains_kernel(const CertifyArgs a)
{
    const int n = *a.list_len;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        const RouterCand c = a.list[i];
        float v = exact_chain(a.x + (size_t)c.t * a.H, a.wrt + (size_t)c.e * a.H, a.H);
        if (a.bias) v = __fadd_rn(v, a.bias[c.e]);
        a.ex[(size_t)c.t * a.E + c.e] = v;
        if (!(fabsf(v - c.v) <= c.d)) atomicCAS(a.status, 0, MOE_ERR_ROUTER_BOUND);
    }
}

// C3: top-k (larger exact value first, lower index on ties) and softmax among each
// token's candidates, one warp per token; the candidates' values are loaded once.
template <int MAXV>
__global__ void __launch_bounds__(256) router_select_kernel(const CertifyArgs a)
{
    extern __shared__ float rsel[];  // [warps][k]
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int t = blockIdx.x * (blockDim.x / 32) + warp;
    if (t >= a.T) return;
    float *sv = rsel + (size_t)warp * a.k;
    const int nc = a.ncand[t];
    const int *cand = a.cand + (size_t)t * a.E;
    const float *ex = a.ex + (size_t)t * a.E;
    int ce[MAXV];
    float cv[MAXV];
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
        const int c = lane + 32 * i;
        ce[i] = c < nc ? cand[c] : INT_MAX;
    }
#pragma unroll
    for (int i = 0; i < MAXV; ++i) cv[i] = ce[i] != INT_MAX ? ex[ce[i]] : 0.0f;
    for (int j = 0; j < a.k; ++j) {
        float bv = 0.0f;
        int be = INT_MAX, bi = -1;
#pragma unroll
        for (int i = 0; i < MAXV; ++i)
            if (ranks_before(cv[i], ce[i], bv, be)) {
                bv = cv[i];
                be = ce[i];
                bi = i;
            }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oe = __shfl_xor_sync(0xffffffffu, be, off);
            if (ranks_before(ov, oe, bv, be)) {
                bv = ov;
                be = oe;
            }
        }
#pragma unroll
        for (int i = 0; i < MAXV; ++i)
            if (i == bi && ce[i] == be) ce[i] = INT_MAX;  // taken
        if (lane == 0) {
            a.idx[(size_t)t * a.k + j] = be;
            sv[j] = bv;
        }
    }
    __syncwarp();
    const float m = sv[0];
    float s = 0.0f;
    for (int j = lane; j < a.k; j += 32) s += expf(sv[j] - m);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    for (int j = lane; j < a.k; j += 32) a.gate[(size_t)t * a.k + j] = expf(sv[j] - m) / s;
}

template <int MAXV>
cudaError_t launch_candidates(const CertifyArgs &a, cudaStream_t st)
{
    router_candidates_kernel<MAXV><<<(a.T + 7) / 8, 256, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

bool small_route_permute_ok(const moe_dims_t &d)
{
    return d.T <= 32 && d.E % 8 == 0 && d.H % 128 == 0 && (long)d.T * d.top_k <= 4096;
}

cudaError_t launch_route_permute_small(const moe_dims_t &d, const __nv_bfloat16 *x, const __nv_bfloat16 *wr,
                                       const float *bias, float *logits, int32_t *idx, float *gate,
                                       int32_t *offsets, int32_t *s2f, int32_t *f2s, int32_t *tiles,
                                       int32_t *ntiles, WsHeader *hdr, cudaStream_t st)
{
    SmallRouteOut o{logits, idx, gate, offsets, s2f, f2s, tiles, ntiles, hdr->counter, 7, &hdr->status};
    cudaError_t e;
    if (d.T <= 16) {
        using L = SmallTile<16, 8, 128, 16>;
        auto kern = route_logits_pipe_kernel<16, 8, 128, 16>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
        if (e != cudaSuccess) return e;
        kern<<<(d.E + 7) / 8, L::NT, L::SMEM, st>>>(x, wr, bias, d.T, d.H, d.E, logits);
    } else {
        using L = SmallTile<32, 8, 128, 16>;
        auto kern = route_logits_pipe_kernel<32, 8, 128, 16>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
        if (e != cudaSuccess) return e;
        kern<<<(d.E + 7) / 8, L::NT, L::SMEM, st>>>(x, wr, bias, d.T, d.H, d.E, logits);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int warps = d.T < 4 ? 4 : d.T;
    const size_t smem = ((size_t)warps * d.top_k + d.E + 64) * 4;
    const int vpl = (d.E + 31) / 32;
    auto launch = [&](auto kern) {
        if (smem > 48 * 1024) {
            cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (r != cudaSuccess) return r;
        }
        kern<<<1, warps * 32, smem, st>>>(d.T, d.E, d.top_k, o);
        return cudaGetLastError();
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
    int32_t *status = &hdr->status;
    __nv_bfloat16 *wrt = rs.wrt;
    float *wsq = rs.wsq;
    cudaError_t e;
    const int vpl = (E + 31) / 32;
    if (T > 32) {
        dim3 tg((E + 31) / 32, (H + 31) / 32);
        router_transpose_kernel<<<tg, 256, 0, st>>>(wr, H, E, wrt);
        router_colnorm_kernel<<<(E + 7) / 8, 256, 0, st>>>(wrt, H, E, wsq);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        int ks = 1;
        if ((e = tc_router_logits(x, wrt, T, H, E, logits, hdr, &ks, st)) != cudaSuccess) return e;
        const float u = 5.9604644775390625e-08f;  // 2^-24
        const float eps = ((float)H * u + 256.0f * u + (float)(H / 64 + ks) * u) * 1.01f;
        CertifyArgs a{logits, ks, x, wrt, wsq, bias, T, H, E, k, eps, rs.ncand, rs.cand, rs.list, &hdr->counter[3],
                      logits, idx, gate, status};
        if ((e = cudaMemsetAsync(&hdr->counter[3], 0, sizeof(int32_t), st)) != cudaSuccess) return e;
        if (vpl <= 1) e = launch_candidates<1>(a, st);
        else if (vpl <= 2) e = launch_candidates<2>(a, st);
        else if (vpl <= 4) e = launch_candidates<4>(a, st);
        else if (vpl <= 8) e = launch_candidates<8>(a, st);
        else if (vpl <= 16) e = launch_candidates<16>(a, st);
        else e = launch_candidates<32>(a, st);
        if (e != cudaSuccess) return e;
        router_chains_kernel<<<num_sms() * 8, 128, 0, st>>>(a);
        const size_t ssm = (size_t)8 * k * sizeof(float);
        if (vpl <= 1) router_select_kernel<1><<<(T + 7) / 8, 256, ssm, st>>>(a);
        else if (vpl <= 2) router_select_kernel<2><<<(T + 7) / 8, 256, ssm, st>>>(a);
        else if (vpl <= 4) router_select_kernel<4><<<(T + 7) / 8, 256, ssm, st>>>(a);
        else if (vpl <= 8) router_select_kernel<8><<<(T + 7) / 8, 256, ssm, st>>>(a);
        else if (vpl <= 16) router_select_kernel<16><<<(T + 7) / 8, 256, ssm, st>>>(a);
        else router_select_kernel<32><<<(T + 7) / 8, 256, ssm, st>>>(a);
        return cudaGetLastError();
    }
    // Pick the tile so that enough warps exist to cover the SMs: small batches get
    // one chain per thread, large ones register-blocked 8x4 or 4x4 chains.
    const long tiles64 = (long)((T + 63) / 64) * ((E + 63) / 64);
    if (T <= 16 && E % 8 == 0 && H % 128 == 0)
        e = launch_logits_small<16, 8, 128, 16>(x, wr, bias, T, H, E, logits, st);
    else if (T <= 32 && E % 8 == 0 && H % 128 == 0)
        e = launch_logits_small<32, 8, 128, 16>(x, wr, bias, T, H, E, logits, st);
    else if (T <= 32)
        e = launch_logits<16, 16, 1, 1, 64>(x, wr, bias, T, H, E, logits, st);
    else if (tiles64 * 4 >= 4 * num_sms())
        e = launch_logits<64, 64, 8, 4, 32>(x, wr, bias, T, H, E, logits, st);
    else
        e = launch_logits<32, 64, 4, 4, 32>(x, wr, bias, T, H, E, logits, st);
    if (e != cudaSuccess) return e;
    if (vpl <= 1) return launch_topk<1>(logits, T, E, k, idx, gate, st);
    if (vpl <= 2) return launch_topk<2>(logits, T, E, k, idx, gate, st);
    if (vpl <= 4) return launch_topk<4>(logits, T, E, k, idx, gate, st);
    if (vpl <= 8) return launch_topk<8>(logits, T, E, k, idx, gate, st);
    if (vpl <= 16) return launch_topk<16>(logits, T, E, k, idx, gate, st);
    return launch_topk<32>(logits, T, E, k, idx, gate, st);
}

}  // namespace moe
