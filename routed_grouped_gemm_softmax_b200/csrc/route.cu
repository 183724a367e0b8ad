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
//   operands staged in shared memory as fp32 (bf16 -> fp32 is exact), each
//   thread owning RT x RE independent chains.
// Kernel 2 (route_topk): one warp per token; k rounds of a warp arg-max with the
//   (larger logit, then lower index) order, then the softmax over the k chosen
//   logits with the maximum subtracted.
#include <cfloat>
#include <climits>

#include "moe_internal.h"

namespace moe {
namespace {

constexpr int HC = 32;  // h values staged per step

template <int TT, int TE, int RT, int RE>
__global__ void __launch_bounds__((TT / RT) * (TE / RE))
route_logits_kernel(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ wr,
                    const float *__restrict__ bias, int T, int H, int E, float *__restrict__ logits)
{
    constexpr int NX = TE / RE;           // threads along experts
    constexpr int NT = (TT / RT) * NX;    // threads per CTA
    __shared__ float xs[TT * (HC + 1)];   // [token][h], padded row
    __shared__ __align__(16) float wsm[HC * TE];  // [h][expert]

    const int tid = threadIdx.x;
    const int tx = tid % NX, ty = tid / NX;
    const int t0 = blockIdx.x * TT, e0 = blockIdx.y * TE;

    float acc[RT][RE];
#pragma unroll
    for (int r = 0; r < RT; ++r)
#pragma unroll
        for (int c = 0; c < RE; ++c) acc[r][c] = 0.0f;

    for (int h0 = 0; h0 < H; h0 += HC) {
        __syncthreads();
        for (int i = tid; i < TT * HC; i += NT) {
            const int tt = i / HC, hh = i % HC;
            const int t = t0 + tt, h = h0 + hh;
            xs[tt * (HC + 1) + hh] = (t < T && h < H) ? __bfloat162float(x[(size_t)t * H + h]) : 0.0f;
        }
        for (int i = tid; i < HC * TE; i += NT) {
            const int hh = i / TE, ee = i % TE;
            const int h = h0 + hh, e = e0 + ee;
            wsm[i] = (h < H && e < E) ? __bfloat162float(wr[(size_t)h * E + e]) : 0.0f;
        }
        __syncthreads();
        const int hn = (H - h0) < HC ? (H - h0) : HC;
        // Chains stop at h = H-1: padding columns would add 0*0 terms, which leave
        // the chain unchanged, but the loop bound keeps the chain length exactly H.
        for (int hh = 0; hh < hn; ++hh) {
            float a[RT], b[RE];
#pragma unroll
            for (int r = 0; r < RT; ++r) a[r] = xs[(ty * RT + r) * (HC + 1) + hh];
            if constexpr (RE == 4) {
                const float4 v = *reinterpret_cast<const float4 *>(&wsm[hh * TE + tx * 4]);
                b[0] = v.x; b[1] = v.y; b[2] = v.z; b[3] = v.w;
            } else {
#pragma unroll
                for (int c = 0; c < RE; ++c) b[c] = wsm[hh * TE + tx * RE + c];
            }
#pragma unroll
            for (int r = 0; r < RT; ++r)
#pragma unroll
                for (int c = 0; c < RE; ++c) acc[r][c] = fmaf(a[r], b[c], acc[r][c]);
        }
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

// (v1, e1) ranks before (v2, e2): larger logit first, equal logits -> lower index.
__device__ __forceinline__ bool ranks_before(float v1, int e1, float v2, int e2)
{
    if (e2 == INT_MAX) return e1 != INT_MAX;
    if (e1 == INT_MAX) return false;
    return v1 > v2 || (v1 == v2 && e1 < e2);
}

template <int MAXV>
__global__ void route_topk_kernel(const float *__restrict__ logits, int T, int E, int k,
                                  int32_t *__restrict__ idx, float *__restrict__ gate)
{
    extern __shared__ float sel[];  // [warps][k] chosen logits
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int t = blockIdx.x * (blockDim.x / 32) + warp;
    if (t >= T) return;
    float *sv = sel + (size_t)warp * k;

    float v[MAXV];
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
        const int e = lane + 32 * i;
        v[i] = e < E ? logits[(size_t)t * E + e] : 0.0f;
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
            idx[(size_t)t * k + j] = be;
            sv[j] = bv;
        }
    }
    __syncwarp();
    const float m = sv[0];  // the first choice holds the largest logit
    float s = 0.0f;
    for (int j = lane; j < k; j += 32) s += expf(sv[j] - m);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    for (int j = lane; j < k; j += 32) gate[(size_t)t * k + j] = expf(sv[j] - m) / s;
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

}  // namespace

cudaError_t launch_route(const moe_dims_t &d, const __nv_bfloat16 *x, const __nv_bfloat16 *wr,
                         const float *bias, float *logits, int32_t *idx, float *gate,
                         cudaStream_t st)
{
    const int T = d.T, H = d.H, E = d.E, k = d.top_k;
    if (T <= 32) {
        dim3 grid((T + 15) / 16, (E + 15) / 16);
        route_logits_kernel<16, 16, 1, 1><<<grid, 256, 0, st>>>(x, wr, bias, T, H, E, logits);
    } else {
        dim3 grid((T + 63) / 64, (E + 63) / 64);
        route_logits_kernel<64, 64, 4, 4><<<grid, 256, 0, st>>>(x, wr, bias, T, H, E, logits);
    }
    cudaError_t e = cudaGetLastError();
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
