// Shared pieces of the CUDA-core FP4 GEMV (used by the public-layout kernel of
// the allocation-free entry point, gemv_canonical.cuh) and the ordered
// combine of the per-pair down outputs.
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
        // s with m * 2^-s in [2^14, 2^15): no fp16 overflow for large rows, full
        // fp16 precision for small ones; s in [-100, 113], 0 for a zero, inf or
        // nan maximum (inf/nan propagate as they are)
        int s = 0;
        if (m > 0.0f && m <= 3.4e38f) s = max(-100, (int)((__float_as_uint(m) >> 23) & 0xff) - 127 - 14);
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

template <int NT>
inline size_t gemv_smem_bytes(int K, int TW, int nthreads)
{
    return sizeof(uint32_t) * ((size_t)(K / 2) * NT + (K / 2) / 16 + 1) + sizeof(float) * (size_t)(nthreads / 32) * NT * TW +
           sizeof(int) * NT + 16;
}

// y[t][h] = sum_j w[t][j] * o[pair_row[t*k + j]][h], slot order, fp32 sums, bf16 once;
// o is fp32, or bf16 (O_BF16) as the tensor-core down tiles leave it.
template <bool O_BF16>
__global__ void combine_kernel(const void* __restrict__ o, const float* __restrict__ w,
                               const int32_t* __restrict__ pair_row, int H, int k, __nv_bfloat16* __restrict__ y)
{
    // 8 consecutive outputs per thread: 16-byte loads of o (the library's own buffer);
    // y (the caller's) is written in 4-byte pairs, as before
    const int t = blockIdx.y;
    const int h = 8 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (h >= H) return;
    float acc[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
    for (int j = 0; j < k; ++j) {
        const float wj = w[(size_t)t * k + j];
        const size_t at = (size_t)pair_row[(size_t)t * k + j] * H + h;
        float v[8];
        if (O_BF16) {
            const uint4 q = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(o) + at);
            const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                v[2 * i] = __uint_as_float(qw[i] << 16);
                v[2 * i + 1] = __uint_as_float(qw[i] & 0xffff0000u);
            }
        } else {
            const float4 a = *reinterpret_cast<const float4*>(static_cast<const float*>(o) + at);
            const float4 b = *reinterpret_cast<const float4*>(static_cast<const float*>(o) + at + 4);
            v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
            v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = fmaf(wj, v[i], acc[i]);
    }
    uint32_t* yw = reinterpret_cast<uint32_t*>(y + (size_t)t * H + h);
#pragma unroll
    for (int i = 0; i < 4; ++i) yw[i] = bf16x2_rn(acc[2 * i], acc[2 * i + 1]);
}

}  // namespace fe
