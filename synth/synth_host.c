/*
 * Seeded synthetic inputs on the host, in plain C: the same counter-based
 * generator as synth/__init__.py (the definition) and synth.cu (the device
 * copy), written out once more so that the tests can draw the weights of
 * hundreds of experts in seconds.  Holds no arithmetic of the MoE layer.
 *
 *   mix64      SplitMix64 output function (Steele, Lea and Flood, OOPSLA 2014)
 *   base       mix64(seed * 256 + tensor_id)
 *   draw j     mix64(base + (3 i + j + 1) * 0x9E3779B97F4A7C15), j = 0, 1, 2
 *   z          (sum of the twelve 16-bit fields of the three draws - 393210) / 65536
 *   weight     float32(z) * float32(0.02)
 */
#include <stdint.h>

#define GAMMA 0x9E3779B97F4A7C15ull

static uint64_t mix64(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

static float normal_at(uint64_t base, uint64_t i)
{
    int64_t s = 0;
    for (int j = 0; j < 3; ++j) {
        const uint64_t d = mix64(base + (3 * i + (uint64_t)j + 1) * GAMMA);
        s += (int64_t)(d & 0xffff) + (int64_t)((d >> 16) & 0xffff) + (int64_t)((d >> 32) & 0xffff) +
             (int64_t)((d >> 48) & 0xffff);
    }
    return (float)(s - 393210) / 65536.0f;
}

static uint64_t stream_base(uint64_t seed, uint64_t tid) { return mix64(seed * 256 + tid); }

/* out[a][k][n], a over the listed experts: W_gate (tensor 0) for n < I, W_up
 * (tensor 1) for n >= I, element (e, k, n') at flat index (e*H + k)*I + n'. */
int synth_host_gate_up(float* out, uint64_t seed, int64_t H, int64_t I, const int64_t* experts, int64_t n_experts)
{
    const uint64_t bg = stream_base(seed, 0), bu = stream_base(seed, 1);
    const float sd = 0.02f;
#pragma omp parallel for schedule(static)
    for (int64_t row = 0; row < n_experts * H; ++row) {
        const int64_t a = row / H, k = row % H, e = experts[a];
        float* dst = out + row * 2 * I;
        const uint64_t f0 = (uint64_t)((e * H + k) * I);
        for (int64_t n = 0; n < I; ++n) {
            dst[n] = normal_at(bg, f0 + (uint64_t)n) * sd;
            dst[I + n] = normal_at(bu, f0 + (uint64_t)n) * sd;
        }
    }
    return 0;
}

/* out[a][k][n] = W_down (tensor 2) of expert experts[a], flat index (e*I + k)*H + n. */
int synth_host_down(float* out, uint64_t seed, int64_t I, int64_t H, const int64_t* experts, int64_t n_experts)
{
    const uint64_t b = stream_base(seed, 2);
    const float sd = 0.02f;
#pragma omp parallel for schedule(static)
    for (int64_t row = 0; row < n_experts * I; ++row) {
        const int64_t a = row / I, k = row % I, e = experts[a];
        float* dst = out + row * H;
        const uint64_t f0 = (uint64_t)((e * I + k) * H);
        for (int64_t n = 0; n < H; ++n) dst[n] = normal_at(b, f0 + (uint64_t)n) * sd;
    }
    return 0;
}

/* out[i] = z(seed, tid, first + i) for i < count (unscaled). */
int synth_host_normal(float* out, uint64_t seed, uint64_t tid, uint64_t first, int64_t count)
{
    const uint64_t b = stream_base(seed, tid);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) out[i] = normal_at(b, first + (uint64_t)i);
    return 0;
}
