// Load-time weight handling: the E2M1 packer (float -> codes + bf16 group
// scales) and the re-layout of the packed [E][K/2][N] format into the column
// tiles the projection kernels stream.
//
// "FireEcho Engine", sections "Key Results" (4x compression, BF16 61 GB ->
// FP4 20 GB) and "Speed Optimization History" step 5 (all experts packed into
// one contiguous [E, K//2, N] buffer).
#pragma once

#include "common.cuh"

namespace fe {

// Two float32 ratios -> one byte of E2M1 codes, (lo -> low nibble, hi -> high
// nibble), by the hardware conversion cvt.rn.satfinite.e2m1x2.f32 (round to
// nearest, ties to the even mantissa bit, magnitudes above 6 saturate to 6).
// A zero magnitude comes back as +0 or -0; -0 (code 8) is stored as code 0.
FE_DEV uint32_t e2m1x2_from_f32(float lo, float hi)
{
    uint32_t r;
    asm("{\n\t.reg .b8 b;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b, %2, %1;\n\t"
        "cvt.u32.u8 %0, b;\n\t}"
        : "=r"(r)
        : "f"(lo), "f"(hi));
    if ((r & 0x0f) == 0x08) r &= 0xf0;
    if ((r & 0xf0) == 0x80) r &= 0x0f;
    return r;
}

// One thread per (expert, group of 32 k, column n).
__global__ void pack_kernel(const float* __restrict__ W, int64_t E, int64_t K, int64_t N, uint8_t* __restrict__ codes,
                            uint16_t* __restrict__ scales)
{
    const int64_t G = K / 32;
    const int64_t total = E * G * N;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = i % N;
        const int64_t eg = i / N;           // e * G + g
        const int64_t e = eg / G, g = eg - e * G;
        const float* src = W + ((e * K) + g * 32) * N + n;
        float v[32];
        float mx = 0.0f;
#pragma unroll
        for (int kk = 0; kk < 32; ++kk) {
            v[kk] = src[(int64_t)kk * N];
            mx = fmaxf(mx, fabsf(v[kk]));
        }
        const __nv_bfloat16 sb = __float2bfloat16_rn(__fdiv_rn(mx, 6.0f));
        const uint16_t sbits = __bfloat16_as_ushort(sb);
        scales[eg * N + n] = sbits;
        const float s = __bfloat162float(sb);
        uint8_t* dst = codes + (e * (K / 2) + g * 16) * N + n;
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            uint32_t byte = 0;
            if (s != 0.0f) byte = e2m1x2_from_f32(__fdiv_rn(v[2 * r], s), __fdiv_rn(v[2 * r + 1], s));
            dst[(int64_t)r * N] = (uint8_t)byte;
        }
    }
}

// Re-layout of one matrix family into column tiles (see gemv.cuh):
//   src codes  [E][K/2][N], src scales [E][K/32][N]
//   dst        [E][n_tiles] tiles of tile_bytes = (K/2)*TW + (K/32)*TW*2:
//              codes [16][K/32][TW] -- entry (i, g, j) is source byte row
//              16*g + i (k = 32g + 2i, 32g + 2i + 1) of tile column j, so the
//              16 rows of one 32-k group are (K/32) * TW bytes apart and
//              consecutive groups are adjacent -- then the scales [K/32][TW]
// Tile column j maps to source column col(tile, j): for the fused gate_up
// matrix (TN = TW/2, I = N/2) j < TN -> tile*TN + j (gate), j >= TN ->
// I + tile*TN + j - TN (up); otherwise tile*TW + j.
struct RelayoutParams {
    const uint8_t* src_codes;
    const uint16_t* src_scales;
    uint8_t* dst;
    int64_t E, K, N;
    int TW;
    int gate_up;
};

FE_DEV int64_t relayout_src_col(const RelayoutParams& p, int64_t tile, int64_t j)
{
    if (p.gate_up) {
        const int64_t TN = p.TW / 2, I = p.N / 2;
        return (j < TN) ? tile * TN + j : I + tile * TN + (j - TN);
    }
    return tile * p.TW + j;
}

// One thread per 16 destination bytes (codes) / 8 destination scales.
__global__ void relayout_kernel(RelayoutParams p)
{
    const int64_t n_tiles = p.N / p.TW;
    const int64_t rows = p.K / 2, G = p.K / 32;
    const int64_t tile_bytes = rows * p.TW + G * p.TW * 2;
    const int64_t cchunks = p.E * n_tiles * rows * (p.TW / 16);
    const int64_t schunks = p.E * n_tiles * G * (p.TW / 8);
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < cchunks + schunks; i += stride) {
        if (i < cchunks) {
            const int64_t jc = i % (p.TW / 16);
            int64_t rest = i / (p.TW / 16);
            const int64_t dr = rest % rows;           // destination row = ii * G + g
            rest /= rows;
            const int64_t tile = rest % n_tiles, e = rest / n_tiles;
            const int64_t ii = dr / G, g = dr % G;
            const int64_t r = 16 * g + ii;            // source byte row
            const int64_t col = relayout_src_col(p, tile, 16 * jc);   // 16 consecutive source columns
            const uint4 v = *reinterpret_cast<const uint4*>(p.src_codes + (e * rows + r) * p.N + col);
            *reinterpret_cast<uint4*>(p.dst + (e * n_tiles + tile) * tile_bytes + dr * p.TW + 16 * jc) = v;
        } else {
            const int64_t i2 = i - cchunks;
            const int64_t jc = i2 % (p.TW / 8);
            int64_t rest = i2 / (p.TW / 8);
            const int64_t g = rest % G;
            rest /= G;
            const int64_t tile = rest % n_tiles, e = rest / n_tiles;
            const int64_t col = relayout_src_col(p, tile, 8 * jc);
            const uint4 v = *reinterpret_cast<const uint4*>(p.src_scales + (e * G + g) * p.N + col);
            *reinterpret_cast<uint4*>(p.dst + (e * n_tiles + tile) * tile_bytes + rows * p.TW + (g * p.TW + 8 * jc) * 2) = v;
        }
    }
}

}  // namespace fe
