// Host E2M1 packer: float W [E][K][N] -> codes [E][K/2][N] + bf16 scales
// [E][K/32][N], the load-time quantiser of the "FireEcho Engine" page
// (section "Key Results": 4x compression of the expert weights).
//
// Rule (per group of 32 consecutive k and column n): scale = bf16 round-to-
// nearest-even of float32(max|w| / 6); each code is the E2M1 magnitude nearest
// to float32(w / scale), exact midpoints to the magnitude whose mantissa bit
// is 0 (which is the even magnitude index), magnitudes beyond 6 to 6, zero as
// code 0, sign in bit 3.  An all-zero group stores scale 0 and codes 0.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace fe_host {

static const float kMagnitude[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

static inline uint16_t bf16_rne_bits(float f)
{
    uint32_t u;
    std::memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) return 0x7fc0;
    const uint32_t lsb = (u >> 16) & 1u;
    return (uint16_t)((u + 0x7fffu + lsb) >> 16);
}

static inline float bf16_value(uint16_t b)
{
    const uint32_t u = (uint32_t)b << 16;
    float f;
    std::memcpy(&f, &u, 4);
    return f;
}

static inline uint32_t encode_e2m1(float r)
{
    const float a = std::fabs(r);
    if (!(a > 0.0f)) return 0;
    int i = 7;                              // largest magnitude index with value <= a
    while (i > 0 && kMagnitude[i] > a) --i;
    int m = i;
    if (i < 7) {
        const float mid = 0.5f * (kMagnitude[i] + kMagnitude[i + 1]);   // exact
        if (a > mid || (a == mid && (i & 1))) m = i + 1;
    }
    if (m == 0) return 0;
    return (uint32_t)m | (r < 0.0f ? 8u : 0u);
}

static void pack_range(const float* W, int64_t K, int64_t N, uint8_t* codes, uint16_t* scales, int64_t eg0,
                       int64_t eg1)
{
    const int64_t G = K / 32;
    for (int64_t eg = eg0; eg < eg1; ++eg) {
        const int64_t e = eg / G, g = eg % G;
        for (int64_t n = 0; n < N; ++n) {
            const float* src = W + (e * K + g * 32) * N + n;
            float mx = 0.0f;
            for (int kk = 0; kk < 32; ++kk) mx = std::fmax(mx, std::fabs(src[kk * N]));
            const uint16_t sb = bf16_rne_bits(mx / 6.0f);
            scales[eg * N + n] = sb;
            const float s = bf16_value(sb);
            uint8_t* dst = codes + (e * (K / 2) + g * 16) * N + n;
            for (int r = 0; r < 16; ++r) {
                uint32_t byte = 0;
                if (s != 0.0f) byte = encode_e2m1(src[(2 * r) * N] / s) | (encode_e2m1(src[(2 * r + 1) * N] / s) << 4);
                dst[r * N] = (uint8_t)byte;
            }
        }
    }
}

void pack(const float* W, int64_t E, int64_t K, int64_t N, uint8_t* codes, uint16_t* scales)
{
    const int64_t total = E * (K / 32);
    unsigned nt = std::thread::hardware_concurrency();
    if (nt == 0) nt = 1;
    if ((int64_t)nt > total) nt = (unsigned)(total > 0 ? total : 1);
    std::vector<std::thread> pool;
    for (unsigned t = 0; t < nt; ++t) {
        const int64_t a = total * t / nt, b = total * (t + 1) / nt;
        pool.emplace_back(pack_range, W, K, N, codes, scales, a, b);
    }
    for (auto& th : pool) th.join();
}

// INT2 scalar codes ("FireEcho Engine", sections "Quantization Formats" and
// "FE-XC / INT2 Cold Expert Demotion": a scalar 2-bit format for the coldest
// experts).  Per group of 32 k and column n: scale = bf16(float32(max|w| /
// 1.5)); the code q of r = float32(w / scale) is the nearest of the levels
// q - 1.5 (q = 0..3), an exact midpoint (r = -1, 0, 1) to the level above;
// four codes per byte, the code of k = 4 b + i in bits 2i, 2i + 1 of byte
// row b.  An all-zero group stores scale 0 and codes 2.
static inline uint32_t encode_int2(float r)
{
    if (r < -1.0f) return 0;
    if (r < 0.0f) return 1;
    if (r < 1.0f) return 2;
    return 3;
}

static void pack_int2_range(const float* W, int64_t K, int64_t N, uint8_t* codes, uint16_t* scales, int64_t eg0,
                            int64_t eg1)
{
    const int64_t G = K / 32;
    for (int64_t eg = eg0; eg < eg1; ++eg) {
        const int64_t e = eg / G, g = eg % G;
        for (int64_t n = 0; n < N; ++n) {
            const float* src = W + (e * K + g * 32) * N + n;
            float mx = 0.0f;
            for (int kk = 0; kk < 32; ++kk) mx = std::fmax(mx, std::fabs(src[kk * N]));
            const uint16_t sb = bf16_rne_bits(mx / 1.5f);
            scales[eg * N + n] = sb;
            const float s = bf16_value(sb);
            uint8_t* dst = codes + (e * (K / 4) + g * 8) * N + n;
            for (int r = 0; r < 8; ++r) {
                uint32_t byte = 0;
                for (int i = 0; i < 4; ++i)
                    byte |= (s != 0.0f ? encode_int2(src[(4 * r + i) * N] / s) : 2u) << (2 * i);
                dst[r * N] = (uint8_t)byte;
            }
        }
    }
}

void pack_int2(const float* W, int64_t E, int64_t K, int64_t N, uint8_t* codes, uint16_t* scales)
{
    const int64_t total = E * (K / 32);
    unsigned nt = std::thread::hardware_concurrency();
    if (nt == 0) nt = 1;
    if ((int64_t)nt > total) nt = (unsigned)(total > 0 ? total : 1);
    std::vector<std::thread> pool;
    for (unsigned t = 0; t < nt; ++t) {
        const int64_t a = total * t / nt, b = total * (t + 1) / nt;
        pool.emplace_back(pack_int2_range, W, K, N, codes, scales, a, b);
    }
    for (auto& th : pool) th.join();
}

}  // namespace fe_host
