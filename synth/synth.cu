// Seeded synthetic weights on the GPU: the same counter-based generator as
// synth/__init__.py (SplitMix64 output function on (seed, tensor id, flat
// index), twelve 16-bit uniforms summed into an approximate N(0,1) value that
// is exact in float32, times float32(0.02)), so every value is bit-identical
// to the host generator's.  Holds no arithmetic of the MoE layer.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

__device__ __forceinline__ uint64_t mix64(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

__host__ __device__ inline uint64_t mix64_h(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

__device__ __forceinline__ float normal_at(uint64_t base, uint64_t i)
{
    int64_t s = 0;
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        const uint64_t d = mix64(base + (3 * i + (uint64_t)j + 1) * kGamma);
        s += (int64_t)(d & 0xffff) + (int64_t)((d >> 16) & 0xffff) + (int64_t)((d >> 32) & 0xffff) +
             (int64_t)((d >> 48) & 0xffff);
    }
    return (float)(s - 393210) / 65536.0f;
}

// dst[(e*H + k)*2I + n]: gate (tensor 0) for n < I, up (tensor 1) for n >= I
__global__ void gate_up_kernel(float* dst, uint64_t base_g, uint64_t base_u, int64_t E, int64_t H, int64_t I)
{
    const int64_t total = E * H * 2 * I;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = i % (2 * I), ek = i / (2 * I);
        const bool up = n >= I;
        const int64_t flat = ek * I + (up ? n - I : n);
        dst[i] = __fmul_rn(normal_at(up ? base_u : base_g, (uint64_t)flat), 0.02f);
    }
}

// dst[i] = normal(seed, tid, i) * scale for i < count
__global__ void plain_kernel(float* dst, uint64_t base, int64_t count, float scale)
{
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < count; i += (int64_t)gridDim.x * blockDim.x)
        dst[i] = __fmul_rn(normal_at(base, (uint64_t)i), scale);
}

uint64_t stream_base(uint64_t seed, uint64_t tid) { return mix64_h(seed * 256 + tid); }

}  // namespace

extern "C" {

// Unquantised fused gate_up weights [E][H][2I] (float32) of a layer seed.
int fe_synth_gate_up(float* dst, uint64_t seed, int64_t E, int64_t H, int64_t I, void* stream)
{
    gate_up_kernel<<<148 * 16, 256, 0, (cudaStream_t)stream>>>(dst, stream_base(seed, 0), stream_base(seed, 1), E, H,
                                                                 I);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

// Unquantised down weights [E][I][H] (float32) of a layer seed (tensor 2).
int fe_synth_down(float* dst, uint64_t seed, int64_t E, int64_t I, int64_t H, void* stream)
{
    plain_kernel<<<148 * 16, 256, 0, (cudaStream_t)stream>>>(dst, stream_base(seed, 2), E * I * H, 0.02f);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

// Approximate N(0,1) * scale for flat indices 0..count-1 of (seed, tensor id).
int fe_synth_normal(float* dst, uint64_t seed, uint64_t tid, int64_t count, float scale, void* stream)
{
    plain_kernel<<<148 * 16, 256, 0, (cudaStream_t)stream>>>(dst, stream_base(seed, tid), count, scale);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // extern "C"
