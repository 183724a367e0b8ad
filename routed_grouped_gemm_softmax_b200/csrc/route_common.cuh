// route_common.cuh -- device helpers shared by the router kernels (route.cu and
// route_certified.cu): cp.async staging, the fp32 chain step with bf16 operands,
// and the warp top-k with the router's order (larger logit first, equal logits ->
// lower expert index).
#pragma once
#include <climits>
#include <cstdint>

#include <cuda_bf16.h>

namespace moe {

__device__ __forceinline__ void cp_async16(void *dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// One step of the logit chain, acc = fma(a, b, acc) with a and b bf16: the mixed
// precision fma of sm_100 widens both operands exactly and rounds once to fp32, so
// it equals fmaf((float)a, (float)b, acc) bit for bit.
__device__ __forceinline__ float chain_step(uint16_t a, uint16_t b, float acc)
{
    asm("fma.rn.f32.bf16 %0, %1, %2, %0;" : "+f"(acc) : "h"(a), "h"(b));
    return acc;
}

// Two steps from a packed pair of a values (lower address first) and two b values.
__device__ __forceinline__ float chain_step2(uint32_t a2, uint16_t b0, uint16_t b1, float acc)
{
    asm("{\n\t.reg .b16 al, ah;\n\tmov.b32 {al, ah}, %1;\n\t"
        "fma.rn.f32.bf16 %0, al, %2, %0;\n\tfma.rn.f32.bf16 %0, ah, %3, %0;\n\t}"
        : "+f"(acc)
        : "r"(a2), "h"(b0), "h"(b1));
    return acc;
}

// Two steps from packed pairs of both operands.
__device__ __forceinline__ float chain_step2x2(uint32_t a2, uint32_t b2, float acc)
{
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, al, bl, %0;\n\tfma.rn.f32.bf16 %0, ah, bh, %0;\n\t}"
        : "+f"(acc)
        : "r"(a2), "r"(b2));
    return acc;
}

// Eight steps from 16-byte vectors of both operands.
__device__ __forceinline__ float chain_step8(const uint4 &a, const uint4 &b, float acc)
{
    acc = chain_step2x2(a.x, b.x, acc);
    acc = chain_step2x2(a.y, b.y, acc);
    acc = chain_step2x2(a.z, b.z, acc);
    return chain_step2x2(a.w, b.w, acc);
}

// Unsigned key with the order of the fp32 values (finite or infinite): larger value
// -> larger key; -0 is folded onto +0 so equal logits get equal keys.  Never 0.
__device__ __forceinline__ uint32_t order_key(float v)
{
    const uint32_t u = __float_as_uint(v + 0.0f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Warp top-k: lane l holds the values of experts l, l+32, ... (MAXV of them; key 0
// marks an empty or invalid slot).  Round j picks the largest key, the lowest expert
// index among equal keys, returns it to every lane in e_out[j] and its value in
// v_out[j] (j < k), and removes it.  At least k valid slots must exist.
template <int MAXV>
__device__ __forceinline__ void warp_topk(uint32_t (&key)[MAXV], const float (&val)[MAXV], int k, int *e_out,
                                          float *v_out)
{
    const int lane = threadIdx.x % 32;
    for (int j = 0; j < k; ++j) {
        uint32_t bk = 0;
        float bv = 0.0f;
        int be = INT_MAX;
#pragma unroll
        for (int i = 0; i < MAXV; ++i)
            if (key[i] > bk) {  // strict: the lowest index of the lane keeps equal keys
                bk = key[i];
                bv = val[i];
                be = lane + 32 * i;
            }
        const uint32_t m = __reduce_max_sync(0xffffffffu, bk);
        const int e = static_cast<int>(
            __reduce_min_sync(0xffffffffu, (bk == m && bk != 0u) ? static_cast<unsigned>(be) : 0xffffffffu));
        const float v = __shfl_sync(0xffffffffu, bv, e & 31);
#pragma unroll
        for (int i = 0; i < MAXV; ++i)
            if (lane + 32 * i == e) key[i] = 0u;
        if (lane == 0) {
            e_out[j] = e;
            v_out[j] = v;
        }
    }
    __syncwarp();
}

}  // namespace moe
