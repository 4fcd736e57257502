// Grouped FP4 GEMV that reads the packed weights in their public format,
// [E][K/2][N] codes and [E][K/32][N] bf16 scales, without any re-layout.
// Used by the allocation-free entry point, whose caller owns the weight
// buffers; the arithmetic is that of gemv.cuh (E2M1 decoded in registers by
// cvt.rn.f16x2.e2m1x2, fp16 x fp16 products accumulated in fp32, one group
// scale per 32 k, SwiGLU in the gate_up epilogue).
//
// A CTA owns one column tile of one routed expert: TW columns (for gate_up
// TW/2 gate columns and the TW/2 up columns of the same outputs); thread
// (chunk c of 16 columns, group g of 32 k) loads the 16 byte rows 16g..16g+15
// of its 16 columns, each 16 bytes, rows N bytes apart.
#pragma once

#include "common.cuh"
#include "gemv.cuh"

namespace fe {

struct CanonParams {
    const uint8_t* codes;     // [E][K/2][N]
    const uint16_t* scales;   // [E][K/32][N] (bf16 bits)
    int K, N;                 // reduction length, columns of the matrix
    int TW;                   // tile width (gate_up: TW/2 gate + TW/2 up columns)
    int n_tiles;
    int N_out;                // I for gate_up (act row), H for down (o row)
    const int32_t* offsets;
    const int32_t* active;
    const int32_t* n_active;
    const int32_t* sorted_pair;
    int top_k;
    const uint16_t* x;
    const float* act_in;
    float* out;
};

template <bool GATE_UP>
FE_DEV int canon_col(const CanonParams& p, int tile, int c)
{
    const int C = p.TW / 16;
    if (GATE_UP) {
        const int TN = p.TW / 2, I = p.N / 2;
        return (c < C / 2) ? tile * TN + 16 * c : I + tile * TN + 16 * (c - C / 2);
    }
    return tile * p.TW + 16 * c;
}

// blockDim.x = roundup32(C * G) <= 256; grid.x = max_active * n_tiles.
// Dynamic shared memory as gemv_kernel: xs | red [nwarps][NT][TW] | shift[NT]
template <int NT, bool GATE_UP>
__global__ void __launch_bounds__(256) gemv_canonical_kernel(CanonParams p)
{
    extern __shared__ __align__(16) uint32_t gsm[];
    const int a = blockIdx.x / p.n_tiles;
    const int tile = blockIdx.x - a * p.n_tiles;
    if (a >= *p.n_active) return;
    const int e = p.active[a];
    const int pos0 = p.offsets[e], npos = p.offsets[e + 1] - pos0;

    const int K = p.K, TW = p.TW, C = TW / 16, G = K / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    const int c = tid % C, g = tid / C;
    const bool valid = g < G;

    uint32_t* xs = gsm;
    float* red = reinterpret_cast<float*>(gsm + xs_words<NT>(K));
    int* shift = reinterpret_cast<int*>(red + nwarps * NT * TW);

    const int col = canon_col<GATE_UP>(p, tile, c);
    const uint8_t* wt = p.codes + (size_t)e * (K / 2) * p.N + col;
    const uint16_t* st = p.scales + ((size_t)e * G + g) * p.N + col;
    uint4 q[16];
    float sc[16];
    if (valid) {
#pragma unroll
        for (int i = 0; i < 16; ++i) q[i] = ldg_stream(wt + (size_t)(16 * g + i) * p.N);
        const uint4 s0 = *reinterpret_cast<const uint4*>(st);
        const uint4 s1 = *reinterpret_cast<const uint4*>(st + 8);
        const uint32_t sw[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            sc[2 * i] = bf16_bits_to_f32((uint16_t)(sw[i] & 0xffff));
            sc[2 * i + 1] = bf16_bits_to_f32((uint16_t)(sw[i] >> 16));
        }
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) q[i] = make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int i = 0; i < 16; ++i) sc[i] = 0.0f;
    }

    GemvParams gp{};   // the staging helper reads only these fields
    gp.K = K;
    gp.sorted_pair = p.sorted_pair;
    gp.top_k = p.top_k;
    gp.x = p.x;
    gp.act_in = p.act_in;

    for (int c0 = 0; c0 < npos; c0 += NT) {
        const int nt = min(NT, npos - c0);
        stage_inputs<NT, GATE_UP>(gp, pos0 + c0, nt, xs, shift, red);
        float acc[NT][16];
#pragma unroll
        for (int tok = 0; tok < NT; ++tok)
#pragma unroll
            for (int j = 0; j < 16; ++j) acc[tok][j] = 0.0f;
        if (valid) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                uint32_t x2[NT];
#pragma unroll
                for (int tok = 0; tok < NT; ++tok) x2[tok] = xs[xs_index<NT>(16 * g + i, tok)];
                const uint32_t words[4] = {q[i].x, q[i].y, q[i].z, q[i].w};
#pragma unroll
                for (int wd = 0; wd < 4; ++wd) {
                    uint32_t h[4];
                    e2m1x8_to_f16x2x4(words[wd], h);
#pragma unroll
                    for (int b = 0; b < 4; ++b)
#pragma unroll
                        for (int tok = 0; tok < NT; ++tok)
                            acc[tok][4 * wd + b] = fma2_f16_f32(h[b], x2[tok], acc[tok][4 * wd + b]);
                }
            }
        }
#pragma unroll
        for (int tok = 0; tok < NT; ++tok) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                float v = acc[tok][j] * sc[j];
                for (int o = C; o < 32; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                acc[tok][j] = v;
            }
            if (lane < C) {
#pragma unroll
                for (int j = 0; j < 16; ++j) red[(warp * NT + tok) * TW + 16 * lane + j] = acc[tok][j];
            }
        }
        __syncthreads();
        if (GATE_UP) {
            const int TN = TW / 2;
            for (int i = tid; i < NT * TN; i += blockDim.x) {
                const int tok = i / TN, n = i - tok * TN;
                if (tok >= nt) continue;
                float gsum = 0.0f, usum = 0.0f;
                for (int w = 0; w < nwarps; ++w) {
                    gsum += red[(w * NT + tok) * TW + n];
                    usum += red[(w * NT + tok) * TW + TN + n];
                }
                const float m = __uint_as_float((uint32_t)(127 + shift[tok]) << 23);
                p.out[(size_t)(pos0 + c0 + tok) * p.N_out + tile * TN + n] = silu_mul(gsum * m, usum * m);
            }
        } else {
            for (int i = tid; i < NT * TW; i += blockDim.x) {
                const int tok = i / TW, n = i - tok * TW;
                if (tok >= nt) continue;
                float s = 0.0f;
                for (int w = 0; w < nwarps; ++w) s += red[(w * NT + tok) * TW + n];
                const float m = __uint_as_float((uint32_t)(127 + shift[tok]) << 23);
                p.out[(size_t)(pos0 + c0 + tok) * p.N_out + tile * TW + n] = s * m;
            }
        }
        __syncthreads();
    }
}

}  // namespace fe
