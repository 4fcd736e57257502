// Load-time weight handling: the E2M1 packer (float -> codes + bf16 group
// scales) and the re-layout of the packed [E][K/2][N] format into the column
// tiles the projection kernels stream.
//
// "FireEcho Engine", sections "Key Results" (4x compression, BF16 61 GB ->
// FP4 20 GB) and "Speed Optimization History" step 5 (all experts packed into
// one contiguous [E, K//2, N] buffer).
#pragma once

#include "common.cuh"
#include "mma.cuh"

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

// INT2 scalar codes (the host packer's rule: scale bf16(max|w| / 1.5) per 32
// along K, the nearest level q - 1.5, midpoints to the level above, four codes
// per byte, the code of k = 4 b + i in bits 2i of byte row b).  One thread per
// (expert, group of 32 k, column n).
FE_DEV uint32_t int2_from_ratio(float r) { return r < -1.0f ? 0u : r < 0.0f ? 1u : r < 1.0f ? 2u : 3u; }

__global__ void pack_int2_kernel(const float* __restrict__ W, int64_t E, int64_t K, int64_t N,
                                 uint8_t* __restrict__ codes, uint16_t* __restrict__ scales)
{
    const int64_t G = K / 32;
    const int64_t total = E * G * N;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = i % N;
        const int64_t eg = i / N;
        const int64_t e = eg / G, g = eg - e * G;
        const float* src = W + ((e * K) + g * 32) * N + n;
        float v[32];
        float mx = 0.0f;
#pragma unroll
        for (int kk = 0; kk < 32; ++kk) {
            v[kk] = src[(int64_t)kk * N];
            mx = fmaxf(mx, fabsf(v[kk]));
        }
        const __nv_bfloat16 sb = __float2bfloat16_rn(__fdiv_rn(mx, 1.5f));
        scales[eg * N + n] = __bfloat16_as_ushort(sb);
        const float s = __bfloat162float(sb);
        uint8_t* dst = codes + (e * (K / 4) + g * 8) * N + n;
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            uint32_t byte = 0;
#pragma unroll
            for (int q = 0; q < 4; ++q) byte |= (s != 0.0f ? int2_from_ratio(__fdiv_rn(v[4 * r + q], s)) : 2u) << (2 * q);
            dst[(int64_t)r * N] = (uint8_t)byte;
        }
    }
}

// Re-layout of one expert matrix family into fragment-ordered column blocks.
//
// A block is 16 columns x K of one expert matrix (the A operand of a
// tensor-core mma.m16n8k16 whose 16 rows are the block's columns and whose K
// is the reduction), stored as one contiguous 9K-byte run:
//   codes  K/64 quads of 512 bytes: byte 16*L + 4*s + j of quad q is the
//          source byte (k-pair row 8*(4q+s) + t + 4*(j>>1), column g + 8*(j&1))
//          with lane L = 4g + t; so lane L of a warp finds, in one 16-byte
//          word, its four A-fragment registers for the four 16-k steps of the
//          quad, each register one byte = (w[k even], w[k odd]) of one column;
//   scales K/32 groups of 8 words: word g of group G holds the bf16 scales of
//          columns g (low half) and g + 8 (high half), the two rows of the
//          mma accumulator a lane owns.
// For the fused gate_up matrix the block of gate columns [16j, 16j+16) is
// followed by the block of up columns [I+16j, I+16j+16), so one gate_up unit
// (both halves of 16 act columns) is one contiguous 18K-byte run.
struct RelayoutParams {
    const uint8_t* src_codes;   // [E][K/2][N]
    const uint16_t* src_scales; // [E][K/32][N]
    uint8_t* dst;               // [E][N/16] blocks of 9K bytes
    int64_t E, K, N;
    int gate_up;
};

FE_DEV int64_t relayout_block_col0(const RelayoutParams& p, int64_t blk)
{
    if (p.gate_up) {
        const int64_t I = p.N / 2, j = blk >> 1;
        return (blk & 1) ? I + 16 * j : 16 * j;
    }
    return 16 * blk;
}

// One thread per destination 4-byte word (codes) or scale word.
__global__ void relayout_kernel(RelayoutParams p)
{
    const int64_t nblk = p.N / 16, K = p.K;
    const int64_t blk_bytes = 9 * K;
    const int64_t cwords = K / 8;     // 8K bytes of codes -> 2K words; per block: K/64 quads * 128 words
    const int64_t code_words = (K / 64) * 128;
    const int64_t scale_words = (K / 32) * 8;
    const int64_t per_blk = code_words + scale_words;
    (void)cwords;
    const int64_t total = p.E * nblk * per_blk;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += stride) {
        const int64_t w = i % per_blk;
        const int64_t eb = i / per_blk;            // e * nblk + blk
        const int64_t e = eb / nblk, blk = eb % nblk;
        const int64_t col0 = relayout_block_col0(p, blk);
        uint32_t v = 0;
        uint8_t* dst = p.dst + eb * blk_bytes;
        if (w < code_words) {
            const int64_t q = w / 128, r = w % 128;
            const int L = (int)(r / 4), s = (int)(r % 4);
            const int g = L >> 2, t = L & 3;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int64_t kp = 8 * (4 * q + s) + t + 4 * (j >> 1);
                const int64_t col = col0 + g + 8 * (j & 1);
                const uint32_t byte = p.src_codes[(e * (K / 2) + kp) * p.N + col];
                v |= byte << (8 * j);
            }
            *reinterpret_cast<uint32_t*>(dst + 512 * q + 16 * L + 4 * s) = v;
        } else {
            const int64_t ws = w - code_words;
            const int64_t G = ws / 8;
            const int g = (int)(ws % 8);
            const uint32_t lo = p.src_scales[(e * (K / 32) + G) * p.N + col0 + g];
            const uint32_t hi = p.src_scales[(e * (K / 32) + G) * p.N + col0 + g + 8];
            *reinterpret_cast<uint32_t*>(dst + 8 * K + 4 * ws) = lo | (hi << 16);
        }
    }
}

// Re-layout of the down matrices into row groups for the single-launch decode
// kernel, which multiplies 16 act values of one expert (the act columns a CTA
// computed) by the 16 matching rows of W_dn for every output column h.  Per
// expert, per group of 32 rows i (one scale group along K = I), one
// contiguous run of 18H bytes:
//   [codes of rows 32g .. 32g+15][scales of group g][codes of rows 32g+16 .. 32g+31]
// so a unit of 16 rows is one contiguous 10H-byte copy (its codes and the
// group's scales, in either order) and two units of one group are one 18H copy.
// Codes of 16 rows x H columns, in the order of the mma.m16n8k16 A fragment
// whose 16 rows are 16 output columns h and whose K is the 16 rows i: byte
// 16L + 4s + j of quad q (512 bytes) belongs to column tile t = 4q + s (16
// columns), lane L = 4g + c, and holds the source byte of row pair c + 4(j>>1)
// (rows 2c, 2c+1, or 2c+8, 2c+9 of the 16) at column 16t + g + 8(j&1).
// Scales: word g of column tile t (8 words per tile) holds the bf16 scales of
// columns 16t + g (low half) and 16t + g + 8 (high half).
struct RowRelayoutParams {
    const uint8_t* src_codes;    // [E][I/2][H]
    const uint16_t* src_scales;  // [E][I/32][H]
    uint8_t* dst;                // [E][I/32] groups of 18H bytes
    int64_t E, I, H;
};

// One thread per destination 4-byte word.
__global__ void relayout_rows_kernel(RowRelayoutParams p)
{
    const int64_t H = p.H, G = p.I / 32;
    const int64_t half_words = 2 * H;           // 8H bytes of codes
    const int64_t scale_words = H / 2;          // 2H bytes of scales
    const int64_t per_group = 2 * half_words + scale_words;
    const int64_t total = p.E * G * per_group;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += stride) {
        const int64_t w = i % per_group, eg = i / per_group;   // eg = e * G + g
        const int64_t e = eg / G, g = eg % G;
        uint8_t* dst = p.dst + eg * 18 * H;
        if (w < half_words || w >= half_words + scale_words) {
            const int half = w < half_words ? 0 : 1;
            const int64_t wc = half == 0 ? w : w - half_words - scale_words;
            const int64_t q = wc / 128, r = wc % 128;
            const int L = (int)(r / 4), sidx = (int)(r % 4);
            const int gg = L >> 2, c = L & 3;
            const int64_t tile = 4 * q + sidx;
            const int64_t row_pair0 = (32 * g + 16 * half) / 2;   // first byte row of the 16 rows
            uint32_t v = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int64_t krow = row_pair0 + c + 4 * (j >> 1);
                const int64_t col = 16 * tile + gg + 8 * (j & 1);
                v |= (uint32_t)p.src_codes[(e * (p.I / 2) + krow) * H + col] << (8 * j);
            }
            const int64_t base = half == 0 ? 0 : 10 * H;
            *reinterpret_cast<uint32_t*>(dst + base + 512 * q + 16 * L + 4 * sidx) = v;
        } else {
            const int64_t ws = w - half_words;     // scale word: tile ws / 8, g' = ws % 8
            const int64_t tile = ws / 8, gg = ws % 8;
            const uint16_t* srow = p.src_scales + (e * G + g) * H;
            const uint32_t lo = srow[16 * tile + gg], hi = srow[16 * tile + gg + 8];
            *reinterpret_cast<uint32_t*>(dst + 8 * H + 4 * ws) = lo | (hi << 16);
        }
    }
}

// INT2 column blocks (mma.cuh, int2_block_bytes): the E2M1 blocks' fragment
// order with two bits per code.  Source codes [E][K/4][N] (code of k in bits
// 2(k % 4) of byte row k / 4).  One thread per destination 32-bit word: word
// w (0, 1) of lane L = 4g + t in quad q holds register r = 4 (s & 1) + j of
// k-step s = 2w + (r >> 2): the codes of column g + 8 (j & 1) at k =
// 64q + 16s + 2t + 8 (j >> 1) (bits 2r) and k + 1 (bits 16 + 2r).
FE_DEV uint32_t int2_code(const uint8_t* src, int64_t N, int64_t k, int64_t col)
{
    return (src[(k >> 2) * N + col] >> (2 * (k & 3))) & 3u;
}

__global__ void relayout_int2_kernel(RelayoutParams p)
{
    const int64_t nblk = p.N / 16, K = p.K;
    const int64_t blk_bytes = int2_block_bytes((int)K);
    const int64_t code_words = (K / 64) * 64;
    const int64_t scale_words = (K / 32) * 8;
    const int64_t per_blk = code_words + scale_words;
    const int64_t total = p.E * nblk * per_blk;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += stride) {
        const int64_t w = i % per_blk;
        const int64_t eb = i / per_blk;
        const int64_t e = eb / nblk, blk = eb % nblk;
        const int64_t col0 = relayout_block_col0(p, blk);
        uint8_t* dst = p.dst + eb * blk_bytes;
        if (w < code_words) {
            const int64_t q = w / 64, r64 = w % 64;
            const int L = (int)(r64 / 2), ww = (int)(r64 % 2);
            const int g = L >> 2, t = L & 3;
            const uint8_t* src = p.src_codes + e * (K / 4) * p.N;
            uint32_t v = 0;
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const int s = 2 * ww + (r >> 2), j = r & 3;
                const int64_t col = col0 + g + 8 * (j & 1);
                const int64_t ke = 64 * q + 16 * s + 2 * t + 8 * (j >> 1);
                v |= int2_code(src, p.N, ke, col) << (2 * r);
                v |= int2_code(src, p.N, ke + 1, col) << (16 + 2 * r);
            }
            *reinterpret_cast<uint32_t*>(dst + 256 * q + 8 * L + 4 * ww) = v;
        } else {
            const int64_t ws = w - code_words;
            const int64_t G = ws / 8;
            const int g = (int)(ws % 8);
            const uint32_t lo = p.src_scales[(e * (K / 32) + G) * p.N + col0 + g];
            const uint32_t hi = p.src_scales[(e * (K / 32) + G) * p.N + col0 + g + 8];
            *reinterpret_cast<uint32_t*>(dst + 4 * K + 4 * ws) = lo | (hi << 16);
        }
    }
}

// INT2 W_dn row groups for the decode kernel: per expert and 32 rows, one 10H
// run [codes of rows 0-15 (4H)][scales of the group (2H)][codes of rows 16-31
// (4H)], the row groups of relayout_rows_kernel with two bits per code: word
// w (0, 1) of lane L = 4g + c in quad q holds register r = 4 (s & 1) + j of
// column tile 4q + s, s = 2w + (r >> 2): the codes of rows 2c + 8 (j >> 1)
// (bits 2r) and that + 1 (bits 16 + 2r) of the 16, at column 16 tile + g +
// 8 (j & 1).  Source codes [E][I/4][H].
__global__ void relayout_int2_rows_kernel(RowRelayoutParams p)
{
    const int64_t H = p.H, G = p.I / 32;
    const int64_t half_words = H;          // 4H bytes of codes
    const int64_t scale_words = H / 2;     // 2H bytes of scales
    const int64_t per_group = 2 * half_words + scale_words;
    const int64_t total = p.E * G * per_group;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += stride) {
        const int64_t w = i % per_group, eg = i / per_group;
        const int64_t e = eg / G, g = eg % G;
        uint8_t* dst = p.dst + eg * 10 * H;
        if (w < half_words || w >= half_words + scale_words) {
            const int half = w < half_words ? 0 : 1;
            const int64_t wc = half == 0 ? w : w - half_words - scale_words;
            const int64_t q = wc / 64, r64 = wc % 64;
            const int L = (int)(r64 / 2), ww = (int)(r64 % 2);
            const int gg = L >> 2, c = L & 3;
            const uint8_t* src = p.src_codes + e * (p.I / 4) * H;
            uint32_t v = 0;
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const int s = 2 * ww + (r >> 2), j = r & 3;
                const int64_t tile = 4 * q + s;
                const int64_t col = 16 * tile + gg + 8 * (j & 1);
                const int64_t row = 32 * g + 16 * half + 2 * c + 8 * (j >> 1);
                v |= int2_code(src, H, row, col) << (2 * r);
                v |= int2_code(src, H, row + 1, col) << (16 + 2 * r);
            }
            const int64_t base = half == 0 ? 0 : 6 * H;
            *reinterpret_cast<uint32_t*>(dst + base + 256 * q + 8 * L + 4 * ww) = v;
        } else {
            const int64_t ws = w - half_words;
            const int64_t tile = ws / 8, gg = ws % 8;
            const uint16_t* srow = p.src_scales + (e * G + g) * H;
            const uint32_t lo = srow[16 * tile + gg], hi = srow[16 * tile + gg + 8];
            *reinterpret_cast<uint32_t*>(dst + 4 * H + 4 * ws) = lo | (hi << 16);
        }
    }
}

}  // namespace fe
