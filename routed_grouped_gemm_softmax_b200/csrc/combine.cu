// combine.cu -- gate-weighted combine back to token order.
//
// Each token's output is the sum of its k expert outputs weighted by the gating
// weights (vLLM fused-MoE page, section 02, last stage; FlashMoE, section 2.1,
// "combine").  The k per-assignment rows of token t sit at flat rows t*k .. t*k+k-1
// of y; they are summed in fp32 in ascending j -- an order fixed by the data, so
// the result is bitwise reproducible -- and rounded once to bf16.
#include "moe_internal.h"

namespace moe {
namespace {

__global__ void combine_kernel(const __nv_bfloat16 *__restrict__ y, const float *__restrict__ gate,
                               int T, int H, int k, __nv_bfloat16 *__restrict__ out)
{
    const int t = blockIdx.x;
    for (int c = threadIdx.x; c < H / 8; c += blockDim.x) {
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
        for (int j = 0; j < k; ++j) {
            const float g = gate[(size_t)t * k + j];
            const uint4 v = reinterpret_cast<const uint4 *>(y + ((size_t)t * k + j) * H)[c];
            const __nv_bfloat162 *p = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(p[i]);
                acc[2 * i] = fmaf(g, f.x, acc[2 * i]);
                acc[2 * i + 1] = fmaf(g, f.y, acc[2 * i + 1]);
            }
        }
        uint4 o;
        __nv_bfloat162 *q = reinterpret_cast<__nv_bfloat162 *>(&o);
#pragma unroll
        for (int i = 0; i < 4; ++i) q[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
        reinterpret_cast<uint4 *>(out + (size_t)t * H)[c] = o;
    }
}

}  // namespace

cudaError_t launch_combine(const __nv_bfloat16 *y, const float *gate, int T, int H, int top_k,
                           __nv_bfloat16 *out, cudaStream_t st)
{
    combine_kernel<<<T, 256, 0, st>>>(y, gate, T, H, top_k, out);
    return cudaGetLastError();
}

}  // namespace moe
