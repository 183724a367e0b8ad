// combine.cu -- the gate-weighted combine as its own kernel, for batches whose
// combine would lengthen the down GEMM's epilogue more than it saves: a CTA per
// token, eight columns per thread, the arithmetic of combine.cuh.
#include "combine.cuh"
#include "moe_internal.h"
#include "pdl.cuh"

namespace moe {
namespace {

// A CTA per token; thread c covers columns 8c .. 8c+7 (and c + 256, ...).
__global__ void __launch_bounds__(256) combine_kernel(const __nv_bfloat16 *__restrict__ y,
                                                      const float *__restrict__ gate, int T, int H, int k,
                                                      __nv_bfloat16 *__restrict__ out, int sh_count, int sh_rows0)
{
    pdl_wait();
    pdl_trigger();
    const int t = blockIdx.x;
    for (int c0 = 0; c0 < H; c0 += 256 * 8)
        combine_cols<false>(y, gate, out, t, k, H, c0 + threadIdx.x * 8, sh_count, T, sh_rows0);
}

}  // namespace

cudaError_t launch_combine(const __nv_bfloat16 *y, const float *gate, int T, int H, int top_k,
                           __nv_bfloat16 *out, cudaStream_t st, int sh_count, int sh_rows0)
{
    return launch_pdl(combine_kernel, dim3(T), dim3(256), 0, st, y, gate, T, H, top_k, out, sh_count, sh_rows0);
}

}  // namespace moe
