// Device helpers shared by the fe_moe kernels (sm_100a only).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "fe_moe kernels are written for sm_100a (B200) only"
#endif

#define FE_DEV __device__ __forceinline__

namespace fe {

// Device status bits (same values as the public FE_DEVICE_* macros).
constexpr uint32_t kDevBadExpert = 0x1;
constexpr uint32_t kDevNanLogit = 0x2;
constexpr uint32_t kDevTcTimeout = 0x10;   // a tensor-core tile gave up waiting for its MMAs

// ---------------------------------------------------------------------------
// E2M1 -> f16x2.  One byte holds two codes, the low nibble for the even k.
// cvt.rn.f16x2.e2m1x2 (PTX ISA 8.6, sm_100a) converts both at once and puts
// the low nibble's value in the low half, so each 32-bit result is
// (w[even k], w[odd k]) of one column.  E2M1 values are exact in fp16.
// ---------------------------------------------------------------------------
FE_DEV void e2m1x8_to_f16x2x4(uint32_t w, uint32_t (&h)[4])
{
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(w));
}

// acc += w.lo * x.lo + w.hi * x.hi with fp16 operands, exact products and fp32
// accumulation (fma.rn.f32.f16, PTX ISA 8.6, sm_100+).  w and x are f16x2.
FE_DEV float fma2_f16_f32(uint32_t w, uint32_t x, float acc)
{
    asm("{\n\t.reg .b16 wl, wh, xl, xh;\n\t"
        "mov.b32 {wl, wh}, %1;\n\t"
        "mov.b32 {xl, xh}, %2;\n\t"
        "fma.rn.f32.f16 %0, wl, xl, %0;\n\t"
        "fma.rn.f32.f16 %0, wh, xh, %0;\n\t}"
        : "+f"(acc)
        : "r"(w), "r"(x));
    return acc;
}

FE_DEV float bf16_bits_to_f32(uint16_t b) { return __uint_as_float(((uint32_t)b) << 16); }

FE_DEV float2 f16x2_to_f32x2(uint32_t h)
{
    __half2 v = *reinterpret_cast<__half2*>(&h);
    return __half22float2(v);
}

FE_DEV uint32_t f32x2_to_f16x2_rn(float a, float b)
{
    __half2 v = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
}

FE_DEV float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

FE_DEV float silu_mul(float g, float u)
{
    // silu(g) * u = g / (1 + exp(-g)) * u, CUDA's expf
    return g / (1.0f + expf(-g)) * u;
}

// The same with the fast exponential and division (a few ulp; 0 for g below
// about -88, where exp(-g) overflows).
FE_DEV float silu_mul_fast(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

// Two floats -> bf16x2 (first in the low half), round to nearest even.
FE_DEV uint32_t bf16x2_rn(float lo, float hi)
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

FE_DEV unsigned long long globaltimer_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ld.global.nc with L1 no-allocate: weights are streamed once per launch.
FE_DEV uint4 ldg_stream(const void* p)
{
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

}  // namespace fe
