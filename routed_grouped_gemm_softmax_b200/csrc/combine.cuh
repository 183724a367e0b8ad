// combine.cuh -- gate-weighted combine back to token order: a warp per (token,
// 256-column n-tile), either fused into the down GEMM's epilogue (small batches)
// or as its own kernel (combine.cu) -- the same arithmetic either way.
//
// Each token's output is the sum of its k expert outputs weighted by the gating
// weights (vLLM fused-MoE page, section 02, last stage; FlashMoE, section 2.1,
// "combine").  The k per-assignment rows of token t sit at flat rows t*k .. t*k+k-1
// of y.  Fused: the down GEMM's epilogue writes them one n-tile (256 columns) at a
// time; after writing, each writer thread makes its row visible (__threadfence) and
// counts one arrival for (token, n-tile).  The thread whose arrival completes the
// count hands the (token, n-tile) to its warp, which sums the k rows of those
// columns in fp32 in ascending j -- an order fixed by the data, so the result is
// bitwise reproducible whichever CTA finishes last -- and rounds once to bf16.
#pragma once
#include <cstdint>

#include <cuda_bf16.h>

namespace moe {

// out[t, col .. col+7] = bf16(sum_j gate[t,j] * y[t*k + j, col .. col+7]), fp32 fma in
// ascending j from 0, then (a shared expert, sh_count > 0) + y[sh_rows0 + s*T + t, ..]
// for s ascending, each at gate 1.  Columns at or past N are skipped (N is a
// multiple of 8).
// FUSED: y was written by other CTAs of the running kernel, so its rows are read
// from L2 (ld.global.cg), eight rows' loads in flight at once since a lone warp
// does the work; the standalone kernel relies on its many resident warps instead.
template <bool FUSED>
__device__ __forceinline__ void combine_cols(const __nv_bfloat16 *__restrict__ y, const float *__restrict__ gate,
                                             __nv_bfloat16 *__restrict__ out, int t, int k, int N, int col,
                                             int sh_count = 0, int T = 0, int sh_rows0 = 0)
{
    if (col >= N) return;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
    auto accumulate = [&](float g, const uint4 &v) {
        const __nv_bfloat162 *p = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(p[i]);
            acc[2 * i] = fmaf(g, f.x, acc[2 * i]);
            acc[2 * i + 1] = fmaf(g, f.y, acc[2 * i + 1]);
        }
    };
    if (FUSED) {
        for (int j0 = 0; j0 < k; j0 += 8) {
            float gg[8];
            uint4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (j0 + u < k) {
                    gg[u] = gate[(size_t)t * k + j0 + u];
                    v[u] = __ldcg(reinterpret_cast<const uint4 *>(y + ((size_t)t * k + j0 + u) * N + col));
                }
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (j0 + u < k) accumulate(gg[u], v[u]);
        }
    } else {
        for (int j = 0; j < k; ++j)
            accumulate(gate[(size_t)t * k + j], *reinterpret_cast<const uint4 *>(y + ((size_t)t * k + j) * N + col));
    }
    for (int s = 0; s < sh_count; ++s) {
        const uint4 *p = reinterpret_cast<const uint4 *>(y + ((size_t)sh_rows0 + (size_t)s * T + t) * N + col);
        accumulate(1.0f, FUSED ? __ldcg(p) : *p);
    }
    uint4 o;
    __nv_bfloat162 *q = reinterpret_cast<__nv_bfloat162 *>(&o);
#pragma unroll
    for (int i = 0; i < 4; ++i) q[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
    *reinterpret_cast<uint4 *>(out + (size_t)t * N + col) = o;
}

// Called by a whole warp after its lanes wrote their y rows of n-tile nt (flat row
// `flat`, or `has_row` false): counts the arrivals and runs the combines they
// complete.  cnt is [T, ntiles]; `target` arrivals complete a (token, n-tile) --
// k, plus sh_count for a shared expert, whose rows sh_rows0 + s*T + t follow.
// Not inlined, so its registers do not add to the epilogue's accumulator pressure.
static __device__ __noinline__ void combine_arrive(const __nv_bfloat16 *__restrict__ y, const float *__restrict__ gate,
                                               __nv_bfloat16 *__restrict__ out, int32_t *__restrict__ cnt, int k,
                                               int target, int N, int ntiles, int nt, bool has_row, int flat,
                                               int lane, int sh_count = 0, int T = 0, int sh_rows0 = 0)
{
    const int tok = !has_row ? 0 : (sh_count == 0 || flat < sh_rows0) ? flat / k : (flat - sh_rows0) % T;
    bool last = false;
    if (has_row) {
        __threadfence();  // this thread's y row before its arrival
        last = atomicAdd(cnt + (size_t)tok * ntiles + nt, 1) == target - 1;
    }
    unsigned m = __ballot_sync(0xffffffffu, last);
    if (m == 0u) return;
    __threadfence();  // after the completing arrivals: the other writers' rows are visible
    __syncwarp();     // ... to every lane of the warp
    while (m) {
        const int src = __ffs(m) - 1;
        m &= m - 1u;
        const int t = __shfl_sync(0xffffffffu, tok, src);
        combine_cols<true>(y, gate, out, t, k, N, nt * 256 + lane * 8, sh_count, T, sh_rows0);  // 256 columns
    }
}

}  // namespace moe
