// Tensor-core building blocks shared by the decode and grouped kernels.
//
// The expert weights are the A operand of mma.sync.m16n8k16 (fp16 x fp16 ->
// fp32): the 16 rows of A are 16 output columns of an expert matrix (one
// fragment-ordered block, see pack.cuh), K is the reduction.  Each lane turns
// one byte of E2M1 codes into one A register with cvt.rn.f16x2.e2m1x2 (the
// low nibble, even k, lands in the low half as the fragment requires), so the
// dequantised weights exist only in registers.  The tokens are the N = 8
// columns of B: x (or act) staged in shared memory as fp16 pairs.  E2M1 and
// bf16-derived fp16 values have at most 2 and 8 significant bits, so every
// product is exact and the sums are fp32; the group scale (bf16) multiplies
// each 32-k partial sum in fp32.
#pragma once

#include "common.cuh"

namespace fe {

FE_DEV void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Bytes of one fragment-ordered block of 16 columns and reduction length K.
__host__ __device__ inline uint32_t block_bytes(int K) { return 9u * (uint32_t)K; }

// Row length (32-bit words) of a staged B row of K values: K/2 f16 pairs plus
// 4 words, so that the 8 rows an mma reads start 4 banks apart.
__host__ __device__ inline int brow_words(int K) { return K / 2 + 4; }

// One quad (64 k = 4 mma k-steps = 2 scale groups) of one block against one
// B row per lane: tot += scale * (A . B) for the lane's accumulator slots.
//   blk   : block base in shared memory
//   brow  : this lane's B row (token of mma column n = lane / 4)
//   q     : quad index
FE_DEV void quad_mma(const uint8_t* blk, int K, const uint32_t* brow, int q, int lane, float (&tot)[4])
{
    const int g = lane >> 2, t = lane & 3;
    const uint4 cw = *reinterpret_cast<const uint4*>(blk + 512 * q + 16 * lane);
    const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
    for (int gi = 0; gi < 2; ++gi) {
        float dg[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int ss = 0; ss < 2; ++ss) {
            const int s = 2 * gi + ss;
            const int kp = 8 * (4 * q + s) + t;
            uint32_t a[4];
            e2m1x8_to_f16x2x4(words[s], a);
            mma16816(dg, a, brow[kp], brow[kp + 4]);
        }
        const uint32_t sw = *reinterpret_cast<const uint32_t*>(blk + 8 * K + 4 * ((2 * q + gi) * 8 + g));
        const float slo = bf16_bits_to_f32((uint16_t)(sw & 0xffff)), shi = bf16_bits_to_f32((uint16_t)(sw >> 16));
        tot[0] = fmaf(dg[0], slo, tot[0]);
        tot[1] = fmaf(dg[1], slo, tot[1]);
        tot[2] = fmaf(dg[2], shi, tot[2]);
        tot[3] = fmaf(dg[3], shi, tot[3]);
    }
}

// Same for two blocks (gate and up of one gate_up unit) sharing the B row.
FE_DEV void quad_mma2(const uint8_t* blk0, const uint8_t* blk1, int K, const uint32_t* brow, int q, int lane,
                      float (&tot0)[4], float (&tot1)[4])
{
    const int g = lane >> 2, t = lane & 3;
    const uint4 c0 = *reinterpret_cast<const uint4*>(blk0 + 512 * q + 16 * lane);
    const uint4 c1 = *reinterpret_cast<const uint4*>(blk1 + 512 * q + 16 * lane);
    const uint32_t w0[4] = {c0.x, c0.y, c0.z, c0.w};
    const uint32_t w1[4] = {c1.x, c1.y, c1.z, c1.w};
#pragma unroll
    for (int gi = 0; gi < 2; ++gi) {
        float d0[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        float d1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int ss = 0; ss < 2; ++ss) {
            const int s = 2 * gi + ss;
            const int kp = 8 * (4 * q + s) + t;
            const uint32_t b0 = brow[kp], b1 = brow[kp + 4];
            uint32_t a[4];
            e2m1x8_to_f16x2x4(w0[s], a);
            mma16816(d0, a, b0, b1);
            e2m1x8_to_f16x2x4(w1[s], a);
            mma16816(d1, a, b0, b1);
        }
        const int wo = 4 * ((2 * q + gi) * 8 + g);
        const uint32_t s0 = *reinterpret_cast<const uint32_t*>(blk0 + 8 * K + wo);
        const uint32_t s1 = *reinterpret_cast<const uint32_t*>(blk1 + 8 * K + wo);
        const float s0l = bf16_bits_to_f32((uint16_t)(s0 & 0xffff)), s0h = bf16_bits_to_f32((uint16_t)(s0 >> 16));
        const float s1l = bf16_bits_to_f32((uint16_t)(s1 & 0xffff)), s1h = bf16_bits_to_f32((uint16_t)(s1 >> 16));
        tot0[0] = fmaf(d0[0], s0l, tot0[0]);
        tot0[1] = fmaf(d0[1], s0l, tot0[1]);
        tot0[2] = fmaf(d0[2], s0h, tot0[2]);
        tot0[3] = fmaf(d0[3], s0h, tot0[3]);
        tot1[0] = fmaf(d1[0], s1l, tot1[0]);
        tot1[1] = fmaf(d1[1], s1l, tot1[1]);
        tot1[2] = fmaf(d1[2], s1h, tot1[2]);
        tot1[3] = fmaf(d1[3], s1h, tot1[3]);
    }
}

// ---- INT2 codes ----------------------------------------------------------------------
// An INT2 block (16 columns x K, see pack.cuh) keeps the E2M1 block's fragment
// order with two bits per code: per quad (64 k) 256 bytes, lane L's 8 at 8L;
// word w of them holds the A registers of k-steps 2w and 2w + 1, register
// r = 4 (s & 1) + j in bits 2r, 2r + 1 (the even k's code) and 16 + 2r,
// 17 + 2r (the odd k's code); then the K/32 x 8 scale words as in an E2M1
// block: 5K bytes.  A code q stands for the level q - 1.5.
__host__ __device__ inline uint32_t int2_block_bytes(int K) { return 5u * (uint32_t)K; }

// The 8 A registers of one INT2 word, register r = f16x2 (2 q_even - 3,
// 2 q_odd - 3): the codes go into the mantissa of 1024 (0x6400), giving
// 1024 + 2q, and 1027 is subtracted; all exact.  Twice the level, so the
// group scale is halved to match.
FE_DEV void int2x8_to_f16x2x8(uint32_t w, uint32_t (&a)[8])
{
    const __half2 off = __half2half2(__ushort_as_half((unsigned short)0x6403u));   // 1027
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const uint32_t bits = (r == 0 ? (w << 1) : (w >> (2 * r - 1))) & 0x00060006u;
        const uint32_t v = bits | 0x64006400u;
        const __half2 h = __hsub2(*reinterpret_cast<const __half2*>(&v), off);
        a[r] = *reinterpret_cast<const uint32_t*>(&h);
    }
}

// quad_mma2_b for two INT2 blocks.
FE_DEV void quad_mma2_b_int2(const uint8_t* blk0, const uint8_t* blk1, int K, const uint32_t (&b)[8], int q,
                             int lane, float (&tot0)[4], float (&tot1)[4])
{
    const int g = lane >> 2;
    const uint2 c0 = *reinterpret_cast<const uint2*>(blk0 + 256 * q + 8 * lane);
    const uint2 c1 = *reinterpret_cast<const uint2*>(blk1 + 256 * q + 8 * lane);
#pragma unroll
    for (int gi = 0; gi < 2; ++gi) {   // scale group gi: k-steps 2gi, 2gi + 1 = word gi
        uint32_t a0[8], a1[8];
        int2x8_to_f16x2x8(gi ? c0.y : c0.x, a0);
        int2x8_to_f16x2x8(gi ? c1.y : c1.x, a1);
        float d0[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        float d1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int ss = 0; ss < 2; ++ss) {
            const int s = 2 * gi + ss;
            const uint32_t x0[4] = {a0[4 * ss], a0[4 * ss + 1], a0[4 * ss + 2], a0[4 * ss + 3]};
            const uint32_t x1[4] = {a1[4 * ss], a1[4 * ss + 1], a1[4 * ss + 2], a1[4 * ss + 3]};
            mma16816(d0, x0, b[2 * s], b[2 * s + 1]);
            mma16816(d1, x1, b[2 * s], b[2 * s + 1]);
        }
        const int wo = 4 * ((2 * q + gi) * 8 + g);
        const uint32_t s0 = *reinterpret_cast<const uint32_t*>(blk0 + 4 * K + wo);
        const uint32_t s1 = *reinterpret_cast<const uint32_t*>(blk1 + 4 * K + wo);
        const float s0l = __uint_as_float(s0 << 16) * 0.5f, s0h = __uint_as_float(s0 & 0xffff0000u) * 0.5f;
        const float s1l = __uint_as_float(s1 << 16) * 0.5f, s1h = __uint_as_float(s1 & 0xffff0000u) * 0.5f;
        tot0[0] = fmaf(d0[0], s0l, tot0[0]);
        tot0[1] = fmaf(d0[1], s0l, tot0[1]);
        tot0[2] = fmaf(d0[2], s0h, tot0[2]);
        tot0[3] = fmaf(d0[3], s0h, tot0[3]);
        tot1[0] = fmaf(d1[0], s1l, tot1[0]);
        tot1[1] = fmaf(d1[1], s1l, tot1[1]);
        tot1[2] = fmaf(d1[2], s1h, tot1[2]);
        tot1[3] = fmaf(d1[3], s1h, tot1[3]);
    }
}

// ---- B operands held in registers --------------------------------------------
// A staged row in "fragment order": the 8 words lane (g, t) feeds to the 4
// k-steps of quad q (k-pairs 8(4q+s)+t and 8(4q+s)+t+4, s = 0..3) sit
// together at q*32 + t*8 + 2s + {0, 1}, so a quad's B fragments are two
// 16-byte loads.  Row strides stay K/2 + 4 words (4 banks apart per row).
__host__ __device__ inline uint32_t bfrag_word(uint32_t kp)
{
    return (kp & ~31u) | ((kp & 3u) << 3) | (((kp >> 3) & 3u) << 1) | ((kp >> 2) & 1u);
}

FE_DEV void load_bfrag(const uint32_t* row, int q, int lane, uint32_t (&b)[8])
{
    const uint4 lo = *reinterpret_cast<const uint4*>(row + q * 32 + (lane & 3) * 8);
    const uint4 hi = *reinterpret_cast<const uint4*>(row + q * 32 + (lane & 3) * 8 + 4);
    b[0] = lo.x; b[1] = lo.y; b[2] = lo.z; b[3] = lo.w;
    b[4] = hi.x; b[5] = hi.y; b[6] = hi.z; b[7] = hi.w;
}

// quad_mma / quad_mma2 with the quad's B fragments in registers (b[2s], b[2s+1]
// for k-step s).
FE_DEV void quad_mma_b(const uint8_t* blk, int K, const uint32_t (&b)[8], int q, int lane, float (&tot)[4])
{
    const int g = lane >> 2;
    const uint4 cw = *reinterpret_cast<const uint4*>(blk + 512 * q + 16 * lane);
    const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
    for (int gi = 0; gi < 2; ++gi) {
        float dg[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int ss = 0; ss < 2; ++ss) {
            const int s = 2 * gi + ss;
            uint32_t a[4];
            e2m1x8_to_f16x2x4(words[s], a);
            mma16816(dg, a, b[2 * s], b[2 * s + 1]);
        }
        const uint32_t sw = *reinterpret_cast<const uint32_t*>(blk + 8 * K + 4 * ((2 * q + gi) * 8 + g));
        const float slo = __uint_as_float(sw << 16), shi = __uint_as_float(sw & 0xffff0000u);
        tot[0] = fmaf(dg[0], slo, tot[0]);
        tot[1] = fmaf(dg[1], slo, tot[1]);
        tot[2] = fmaf(dg[2], shi, tot[2]);
        tot[3] = fmaf(dg[3], shi, tot[3]);
    }
}

FE_DEV void quad_mma2_b(const uint8_t* blk0, const uint8_t* blk1, int K, const uint32_t (&b)[8], int q, int lane,
                        float (&tot0)[4], float (&tot1)[4])
{
    const int g = lane >> 2;
    const uint4 c0 = *reinterpret_cast<const uint4*>(blk0 + 512 * q + 16 * lane);
    const uint4 c1 = *reinterpret_cast<const uint4*>(blk1 + 512 * q + 16 * lane);
    const uint32_t w0[4] = {c0.x, c0.y, c0.z, c0.w};
    const uint32_t w1[4] = {c1.x, c1.y, c1.z, c1.w};
#pragma unroll
    for (int gi = 0; gi < 2; ++gi) {
        float d0[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        float d1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int ss = 0; ss < 2; ++ss) {
            const int s = 2 * gi + ss;
            uint32_t a[4];
            e2m1x8_to_f16x2x4(w0[s], a);
            mma16816(d0, a, b[2 * s], b[2 * s + 1]);
            e2m1x8_to_f16x2x4(w1[s], a);
            mma16816(d1, a, b[2 * s], b[2 * s + 1]);
        }
        const int wo = 4 * ((2 * q + gi) * 8 + g);
        const uint32_t s0 = *reinterpret_cast<const uint32_t*>(blk0 + 8 * K + wo);
        const uint32_t s1 = *reinterpret_cast<const uint32_t*>(blk1 + 8 * K + wo);
        const float s0l = __uint_as_float(s0 << 16), s0h = __uint_as_float(s0 & 0xffff0000u);
        const float s1l = __uint_as_float(s1 << 16), s1h = __uint_as_float(s1 & 0xffff0000u);
        tot0[0] = fmaf(d0[0], s0l, tot0[0]);
        tot0[1] = fmaf(d0[1], s0l, tot0[1]);
        tot0[2] = fmaf(d0[2], s0h, tot0[2]);
        tot0[3] = fmaf(d0[3], s0h, tot0[3]);
        tot1[0] = fmaf(d1[0], s1l, tot1[0]);
        tot1[1] = fmaf(d1[1], s1l, tot1[1]);
        tot1[2] = fmaf(d1[2], s1h, tot1[2]);
        tot1[3] = fmaf(d1[3], s1h, tot1[3]);
    }
}

// Power-of-two shift s of a row staged as fp16 (m = max |v| of the row): the
// row is stored as v * 2^-s with m * 2^-s in [2^14, 2^15), so a large row
// cannot overflow and a small one keeps fp16's full precision instead of
// sinking into its subnormal range.  s is clamped to [-100, 113] (both 2^s and
// 2^-s stay normal floats); a zero, infinite or NaN maximum gives s = 0.
FE_DEV int fp16_shift(float m)
{
    if (!(m > 0.0f) || m > 3.4e38f) return 0;
    const int s = (int)((__float_as_uint(m) >> 23) & 0xff) - 127 - 14;
    return s < -100 ? -100 : s;
}

FE_DEV float pow2f(int e) { return __uint_as_float((uint32_t)(127 + e) << 23); }

// One warp stages one row of n values (bf16 bits, or fp32 read through L2)
// as n/2 f16x2 words scaled by 2^-s; returns s.
template <bool BF16>
FE_DEV int warp_stage_row(const void* src, int n, uint32_t* dst, int lane)
{
    float m = 0.0f;
    for (int r = lane; r < n / 2; r += 32) {
        float a, b;
        if (BF16) {
            const uint32_t two = static_cast<const uint32_t*>(src)[r];
            a = bf16_bits_to_f32((uint16_t)(two & 0xffff));
            b = bf16_bits_to_f32((uint16_t)(two >> 16));
        } else {
            const float2 two = __ldcg(static_cast<const float2*>(src) + r);
            a = two.x;
            b = two.y;
        }
        m = fmaxf(m, fmaxf(fabsf(a), fabsf(b)));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const int s = fp16_shift(m);
    const float sc = pow2f(-s);
    for (int r = lane; r < n / 2; r += 32) {
        float a, b;
        if (BF16) {
            const uint32_t two = static_cast<const uint32_t*>(src)[r];
            a = bf16_bits_to_f32((uint16_t)(two & 0xffff));
            b = bf16_bits_to_f32((uint16_t)(two >> 16));
        } else {
            const float2 two = __ldcg(static_cast<const float2*>(src) + r);
            a = two.x;
            b = two.y;
        }
        dst[r] = f32x2_to_f16x2_rn(a * sc, b * sc);
    }
    return s;
}

}  // namespace fe
