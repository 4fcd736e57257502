// Grouped FP4 GEMV for small token counts: the gate_up projection with the
// SwiGLU epilogue, and the down projection.
//
// "FireEcho Engine", section "The Goliath Kernel: Why It's Fast": packed FP4
// bytes are loaded, split into the low and high nibble, multiplied by the
// group scale in registers and accumulated; nothing dequantised is written
// to memory, and the expert id of each work item is read from device memory
// (the routing of route.cuh).  Section "Speed Optimization History": fused
// gate_up (step 2), single-token decode path (step 3), one launch for all
// routed experts (step 4), one contiguous buffer for all experts (step 5).
//
// Weight layout inside the library (re-laid out at load time from the
// [E][K/2][N] byte / [E][K/32][N] scale format): every expert matrix is cut
// into column tiles of TW columns; a tile is one contiguous block of K/2 byte
// rows of TW bytes, byte row r holding k = 2r in the low nibbles and k = 2r+1
// in the high nibbles, stored group-interleaved: [16][K/32][TW], entry
// (i, g) = byte row 16g + i.  A thread owning group g reads its 16 rows with a
// stride of (K/32) * TW bytes, and neighbouring threads (neighbouring groups)
// read neighbouring 16-byte vectors.  The K/32 rows of TW bf16 scales of the
// tile follow its codes, so one tile is one contiguous block.
// For gate_up a tile holds TN gate columns then the TN matching up columns,
// so the SwiGLU epilogue of a tile needs nothing from another tile.
//
// Work split inside a CTA: thread = (chunk c of 16 columns, group g of 32 k),
// C = TW/16 chunks and G = K/32 groups, so every thread owns exactly one
// scale per column.  It loads 16 rows x 16 bytes (all its weights) with
// streaming 128-bit loads up front, converts each byte with
// cvt.rn.f16x2.e2m1x2 and accumulates x[k] * code in fp32 (fma.rn.f32.f16:
// exact products, fp32 sums), applies the group scale once, and the K
// reduction finishes with warp shuffles and one shared-memory pass.
#pragma once

#include "common.cuh"

namespace fe {

struct GemvParams {
    const uint8_t* tiles;     // [E][n_tiles] x {codes [16][K/32][TW], scales bf16 [K/32][TW]}
    int K;                    // reduction length
    int TW;                   // tile width in columns (bytes per row)
    int n_tiles;              // tiles per expert
    int N_out;                // row length of the output (I for gate_up, H for down)
    const int32_t* offsets;   // [E+1]
    const int32_t* active;    // [E]
    const int32_t* n_active;  // [1]
    const int32_t* sorted_pair;
    int top_k;
    const uint16_t* x;        // gate_up input: bf16 [T][K]
    const float* act_in;      // down input: fp32 [P][K] by sorted position
    float* out;               // gate_up: act [P][I]; down: o [P][H], by sorted position
};

// Rows of the staged input: element r holds (v[2r], v[2r+1]) of NT tokens as
// f16x2; one padding word every 16 rows spreads the 8 groups a warp touches
// over different banks.
template <int NT>
FE_DEV int xs_index(int r, int tok) { return r * NT + tok + (r >> 4); }

template <int NT>
FE_DEV int xs_words(int K) { return (K / 2) * NT + (K / 2) / 16 + 1; }

// Stage NT input rows (token chunk) as f16x2 with a per-token power-of-two
// shift so that every value fits fp16; returns nothing, writes shift[tok].
template <int NT, bool GATE_UP>
FE_DEV void stage_inputs(const GemvParams& p, int e_pos0, int nt, uint32_t* xs, int* shift, float* red)
{
    const int tid = threadIdx.x, nthreads = blockDim.x;
    const int K = p.K;
    // 1. max |v| per token
    for (int tok = 0; tok < NT; ++tok) {
        float m = 0.0f;
        if (tok < nt) {
            const int pos = e_pos0 + tok;
            if (GATE_UP) {
                const int t = p.sorted_pair[pos] / p.top_k;
                const uint16_t* xr = p.x + (size_t)t * K;
                for (int i = tid; i < K; i += nthreads) m = fmaxf(m, fabsf(bf16_bits_to_f32(xr[i])));
            } else {
                const float* ar = p.act_in + (size_t)pos * K;
                for (int i = tid; i < K; i += nthreads) m = fmaxf(m, fabsf(ar[i]));
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if ((tid & 31) == 0) red[(tid >> 5) * NT + tok] = m;
    }
    __syncthreads();
    if (tid < NT) {
        float m = 0.0f;
        for (int w = 0; w < nthreads / 32; ++w) m = fmaxf(m, red[w * NT + tid]);
        // smallest s >= 0 with m * 2^-s < 2^15
        int s = 0;
        if (m >= 32768.0f) s = (int)((__float_as_uint(m) >> 23) & 0xff) - 127 - 14;
        if (!(m == m) || m > 3.0e38f) s = 0;  // inf/nan propagate as they are
        shift[tid] = s;
    }
    __syncthreads();
    // 2. convert
    for (int r = tid; r < K / 2; r += nthreads) {
#pragma unroll
        for (int tok = 0; tok < NT; ++tok) {
            float a = 0.0f, b = 0.0f;
            if (tok < nt) {
                const int pos = e_pos0 + tok;
                const float sc = __uint_as_float((uint32_t)(127 - shift[tok]) << 23);
                if (GATE_UP) {
                    const int t = p.sorted_pair[pos] / p.top_k;
                    const uint32_t two = *reinterpret_cast<const uint32_t*>(p.x + (size_t)t * K + 2 * r);
                    a = bf16_bits_to_f32((uint16_t)(two & 0xffff)) * sc;
                    b = bf16_bits_to_f32((uint16_t)(two >> 16)) * sc;
                } else {
                    const float2 two = *reinterpret_cast<const float2*>(p.act_in + (size_t)pos * K + 2 * r);
                    a = two.x * sc;
                    b = two.y * sc;
                }
            }
            xs[xs_index<NT>(r, tok)] = f32x2_to_f16x2_rn(a, b);
        }
    }
    __syncthreads();
}

// blockDim.x = roundup32(C * G) <= 256; grid.x = max_active * n_tiles.
// Dynamic shared memory: xs (f16x2 rows) | red [nwarps][NT][TW] floats | shift[NT]
template <int NT, bool GATE_UP>
__global__ void __launch_bounds__(256) gemv_kernel(GemvParams p)
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

    // this thread's weights: 16 rows x 16 bytes and 16 scales
    const size_t tile_id = (size_t)e * p.n_tiles + tile;
    const uint8_t* wt = p.tiles + tile_id * ((size_t)(K / 2) * TW + (size_t)G * TW * 2);
    const uint16_t* st = reinterpret_cast<const uint16_t*>(wt + (size_t)(K / 2) * TW);
    uint4 q[16];
    float sc[16];
    if (valid) {
#pragma unroll
        for (int i = 0; i < 16; ++i) q[i] = ldg_stream(wt + ((size_t)i * G + g) * TW + 16 * c);
        const uint4 s0 = *reinterpret_cast<const uint4*>(st + (size_t)g * TW + 16 * c);
        const uint4 s1 = *reinterpret_cast<const uint4*>(st + (size_t)g * TW + 16 * c + 8);
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

    for (int c0 = 0; c0 < npos; c0 += NT) {
        const int nt = min(NT, npos - c0);
        stage_inputs<NT, GATE_UP>(p, pos0 + c0, nt, xs, shift, red);
        // partial dot products of this thread's group for every token of the chunk
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
                // reduce over the lanes of this warp that hold the same chunk
                for (int o = C; o < 32; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                acc[tok][j] = v;
            }
            if (lane < C) {
#pragma unroll
                for (int j = 0; j < 16; ++j) red[(warp * NT + tok) * TW + 16 * lane + j] = acc[tok][j];
            }
        }
        __syncthreads();
        // finish the K reduction and write
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

template <int NT>
inline size_t gemv_smem_bytes(int K, int TW, int nthreads)
{
    return sizeof(uint32_t) * ((size_t)(K / 2) * NT + (K / 2) / 16 + 1) + sizeof(float) * (size_t)(nthreads / 32) * NT * TW +
           sizeof(int) * NT + 16;
}

// y[t][h] = sum_j w[t][j] * o[pair_row[t*k + j]][h], slot order, fp32, bf16 once.
__global__ void combine_kernel(const float* __restrict__ o, const float* __restrict__ w,
                               const int32_t* __restrict__ pair_row, int H, int k, __nv_bfloat16* __restrict__ y)
{
    const int t = blockIdx.y;
    const int h = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (h >= H) return;
    float a0 = 0.0f, a1 = 0.0f;
    for (int j = 0; j < k; ++j) {
        const float wj = w[(size_t)t * k + j];
        const float2 v = *reinterpret_cast<const float2*>(o + (size_t)pair_row[(size_t)t * k + j] * H + h);
        a0 = fmaf(wj, v.x, a0);
        a1 = fmaf(wj, v.y, a1);
    }
    *reinterpret_cast<__nv_bfloat162*>(y + (size_t)t * H + h) = __floats2bfloat162_rn(a0, a1);
}

}  // namespace fe
