// fp8_common.cuh -- device helpers of the fp8 kernels (fp8.cu, fp8_swapab.cu): the
// e4m3 quantiser's arithmetic (s = amax/448, codes rounded to nearest even and
// saturated at +-448), SwiGLU's silu, and the kind::f8f6f4 MMA.
#pragma once
#include <cstdint>

#include <cuda_fp8.h>

namespace moe {

__device__ __forceinline__ void record(int32_t *status, int code) { atomicCAS(status, 0, code); }

__device__ __forceinline__ float silu(float a) { return a / (1.0f + __expf(-a)); }

// e4m3 codes of a and b (already divided by the scale), round to nearest even,
// saturated at +-448; a in the low byte.  A negative value that rounds to zero keeps
// its sign (code 0x80), as an IEEE-style conversion does.
__device__ __forceinline__ uint32_t e4m3_pair(float a, float b)
{
    const __nv_fp8x2_storage_t p = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
    return static_cast<uint32_t>(p);
}

__device__ __forceinline__ uint8_t e4m3_one(float a)
{
    return static_cast<uint8_t>(__nv_cvt_float_to_fp8(a, __NV_SATFINITE, __NV_E4M3));
}

// v / s, IEEE-rounded, clamped to the e4m3 range.
__device__ __forceinline__ float qdiv(float v, float s)
{
    return fminf(fmaxf(__fdiv_rn(v, s), -448.0f), 448.0f);
}

// kind::f8f6f4 instruction descriptor: e4m3 A and B (K-major), fp32 accumulator.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N)
{
    return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_e4m3(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
        : "memory");
}

}  // namespace moe
