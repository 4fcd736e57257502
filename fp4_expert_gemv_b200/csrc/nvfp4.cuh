// Block-scaled FP4 (NVFP4) variant of the large-T projections on the
// 5th-generation tensor cores: tcgen05.mma kind::mxf4nvf4 with E4M3 scale
// factors per 16 elements, both operands FP4.
//
// "FireEcho Engine", section "The Goliath Kernel: Why It's Fast": FP4 codes are
// what the matmul reads.  The tensor cores' FP4 rate takes scale factors that
// are E4M3 per 16 elements (or powers of two per 32), so the layer's BF16 group
// scales cannot be fed as they are: this variant re-encodes the weights at
// load and the activations on the fly, and is therefore an approximation of
// the layer (its distance to the exact layer is measured, not bounded by the
// layer's tolerance).  The encoding of a row of K values v:
//
//   g   = amax|v| / 2688               (6 * 448: the row's fp32 scale)
//   s_b = E4M3(amax_b / (6 g))          per block b of 16, nearest, ties even, <= 448
//   q   = E2M1(v * r_b), r_b = 1 / (s_b g)   nearest, ties even, |.| <= 6
//
// every step in fp32 (IEEE division, reciprocal and products, no
// contraction), so that the codes are the same wherever they are computed.  The product of two
// encoded rows is sum_b s_b^x s_b^w sum_k q^x q^w, times g^x g^w: the tensor
// core forms the block-scaled sum, the epilogue multiplies by the row scales.
//
// Operands reach shared memory as ready-made tile images, so one CTA-local
// cp.async.bulk per operand and stage moves them (no tensor map, no
// multicast): a stage holds 256 K elements (128 bytes per row) of
//   A: 128 weight rows, K-major with the 128-byte swizzle (16 KB), then their
//      scale factors in the tensor core's 32 x 16-byte blocks (2 KB);
//   B: 256 token rows, the same (32 KB), then their scale factors (4 KB).
// Weight images are built once per load from the packed layer; token images
// per forward, one 256-row slot per tile of the tile list (tcgen05.cuh).
#pragma once

#include <cuda_fp8.h>

#include "bulk.cuh"
#include "tcgen05.cuh"

namespace fe {

constexpr int kNvM = 128;                              // weight rows per tile (the MMA's M)
constexpr int kNvN = 256;                              // token rows per tile (N <= 256)
constexpr int kNvKc = 256;                             // K elements per stage: 128 bytes per row
constexpr int kNvStages = 4;
constexpr uint32_t kNvACodes = kNvM * 128;             // 16 KB
constexpr uint32_t kNvAChunk = kNvACodes + kNvM * 16;  // + 16 scale factors per row
constexpr uint32_t kNvBCodes = kNvN * 128;             // 32 KB
constexpr uint32_t kNvBChunk = kNvBCodes + kNvN * 16;
constexpr int kNvThreads = 128;
constexpr uint32_t kNvTmemCols = 512;                  // accumulator 256 + 48 per stage for scale factors
constexpr uint32_t kNvSfCols = 48;                     // per stage: A 4 x 4 columns, B 4 x 8 columns

// Dynamic shared memory: alignment slack, the A and B rings, barriers, TMEM slot, flags.
__host__ __device__ inline uint32_t nv_smem_bytes()
{
    return 1024 + kNvStages * (kNvAChunk + kNvBChunk) + 8 * (2 * kNvStages + 1) + 16;
}

// ---- tile-image layout -------------------------------------------------------------
// Byte of row r holding code bytes kb (0..127) of a stage: 16-byte chunks of a
// 128-byte row permuted by the row's index mod 8 (the 128-byte swizzle, with the
// tile at a 1024-byte aligned address).
__host__ __device__ inline uint32_t nv_code_off(int r, int kb)
{
    return (uint32_t)r * 128u + ((uint32_t)((kb >> 4) ^ (r & 7)) << 4) + (uint32_t)(kb & 15);
}

// Scale factor j (0..15: k-block j / 4 of 64, its 16-element block j % 4) of A
// row r (0..127): per k-block a 512-byte block in which 16-byte line r % 32
// holds rows r % 32, +32, +64, +96, four factors each.
__host__ __device__ inline uint32_t nv_sfa_off(int r, int j)
{
    return kNvACodes + 512u * (uint32_t)(j >> 2) + 16u * (uint32_t)(r & 31) + 4u * (uint32_t)(r >> 5) + (uint32_t)(j & 3);
}

// The same for B row n (0..255): per k-block two such blocks, rows 0..127 then 128..255.
__host__ __device__ inline uint32_t nv_sfb_off(int n, int j)
{
    return kNvBCodes + 1024u * (uint32_t)(j >> 2) + 512u * (uint32_t)(n >> 7) + 16u * (uint32_t)(n & 31) +
           4u * (uint32_t)((n >> 5) & 3) + (uint32_t)(j & 3);
}

// gate_up image row R of an expert (0..2I-1) -> its column of the packed [H/2][2I]
// matrix: rows 32b .. 32b+15 are gate columns 16b.., rows 32b+16 .. 32b+31 the up
// columns I + 16b.., so the epilogue finds gate and up of one act column in lanes
// l and l + 16 of one warp.
__host__ __device__ inline int nv_gate_up_column(int R, int I)
{
    const int b = R >> 5, w = R & 31;
    return w < 16 ? 16 * b + w : I + 16 * b + (w - 16);
}

// ---- the encoding ------------------------------------------------------------------
FE_DEV float e4m3_value(uint32_t b)
{
    const uint32_t e = (b >> 3) & 15u, m = b & 7u;
    return e == 0 ? (float)m * 0.001953125f : __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Value of an E2M1 code: magnitudes 0, 0.5, 1, 1.5 (exponent field 0 or 1), then
// 2^(e-1) (1 + m/2); bit 3 is the sign.
FE_DEV float e2m1_value(uint32_t q)
{
    const uint32_t e = (q >> 1) & 3u, m = q & 1u;
    const float mag = e == 0 ? 0.5f * (float)m : (float)(1u << (e - 1)) * (1.0f + 0.5f * (float)m);
    return (q & 8u) ? -mag : mag;
}

// Nearest E4M3 (ties to even) of t >= 0, saturating at 448.
FE_DEV uint32_t e4m3_rn(float t) { return (uint32_t)__nv_cvt_float_to_fp8(t, __NV_SATFINITE, __NV_E4M3) & 0x7Fu; }

// Eight values -> eight E2M1 codes (nearest, ties to even, |.| <= 6) in one
// word, r[i] in bits 4i .. 4i+3.  cvt ... e2m1x2 puts its first source in the
// high nibble.  A zero magnitude is written as code 0 (no negative zero).
FE_DEV uint32_t e2m1x8_rn(const float* r)
{
    uint32_t w;
    asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q3, %8, %7;\n\t"
        "mov.b32 %0, {q0, q1, q2, q3};\n\t}"
        : "=r"(w)
        : "f"(r[0]), "f"(r[1]), "f"(r[2]), "f"(r[3]), "f"(r[4]), "f"(r[5]), "f"(r[6]), "f"(r[7]));
    const uint32_t m = w & 0x77777777u;                                  // magnitudes
    const uint32_t nz = (m | (m >> 1) | (m >> 2)) & 0x11111111u;         // per nibble: magnitude != 0
    return m | (w & (nz << 3));
}

// Row scale g and 6 g from the row's largest magnitude.
FE_DEV void nv_row_scale(float amax, float& g, float& d6)
{
    g = __fdiv_rn(amax, 2688.0f);
    d6 = __fmul_rn(6.0f, g);
}

// One block of 16 values: its scale factor byte and 8 code bytes (two words,
// byte i = elements 2i (low nibble), 2i + 1).
FE_DEV uint32_t nv_encode_block(const float (&v)[16], float g, float d6, uint32_t (&codes)[2])
{
    float ab = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) ab = fmaxf(ab, fabsf(v[i]));
    const uint32_t sb = d6 > 0.0f ? e4m3_rn(__fdiv_rn(ab, d6)) : 0u;
    const float dq = __fmul_rn(e4m3_value(sb), g);
    const float rq = dq > 0.0f ? __frcp_rn(dq) : 0.0f;
    float r[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) r[i] = __fmul_rn(v[i], rq);
    codes[0] = e2m1x8_rn(r);
    codes[1] = e2m1x8_rn(r + 8);
    return sb;
}

FE_DEV void bf16x16_to_f32(const uint16_t* src, float (&v)[16])
{
    const uint4 a = *reinterpret_cast<const uint4*>(src);
    const uint4 b = *reinterpret_cast<const uint4*>(src + 8);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        v[2 * i] = bf16_bits_to_f32((uint16_t)(w[i] & 0xffffu));
        v[2 * i + 1] = bf16_bits_to_f32((uint16_t)(w[i] >> 16));
    }
}

// 16 values of a row: bf16 (two 16-byte loads) or fp32 (four).
template <bool BF16>
FE_DEV void nv_load16(const void* row, int b, float (&v)[16])
{
    if (BF16) {
        bf16x16_to_f32(static_cast<const uint16_t*>(row) + 16 * b, v);
    } else {
        const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(row) + 16 * b);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float4 q = p[i];
            v[4 * i] = q.x; v[4 * i + 1] = q.y; v[4 * i + 2] = q.z; v[4 * i + 3] = q.w;
        }
    }
}

// Rows of bf16 or fp32 values -> NVFP4 in plain row order: codes [R][K/2],
// scale factors [R][K/16], row scales [R].  One warp per row.
template <bool BF16>
__global__ void nvfp4_rows_kernel(const void* src, int R, int K, uint8_t* codes, uint8_t* sf, float* g_out)
{
    const int r = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5), lane = threadIdx.x & 31;
    if (r >= R) return;
    const void* row = BF16 ? (const void*)(static_cast<const uint16_t*>(src) + (size_t)r * K)
                           : (const void*)(static_cast<const float*>(src) + (size_t)r * K);
    float amax = 0.0f;
    for (int b = lane; b < K / 16; b += 32) {
        float v[16];
        nv_load16<BF16>(row, b, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    float g, d6;
    nv_row_scale(amax, g, d6);
    for (int b = lane; b < K / 16; b += 32) {
        float v[16];
        nv_load16<BF16>(row, b, v);
        uint32_t c[2];
        sf[(size_t)r * (K / 16) + b] = (uint8_t)nv_encode_block(v, g, d6, c);
        *reinterpret_cast<uint2*>(codes + (size_t)r * (K / 2) + 8 * b) = make_uint2(c[0], c[1]);
    }
    if (lane == 0) g_out[r] = g;
}

// ---- weight images (once per load) -------------------------------------------------
// Thread per (expert, image row R): the row's K values are the packed layer's
// column n (E2M1 code x bf16 group scale, exact in fp32), read from the plain
// [E][K/2][N] codes and [E][K/32][N] scales.  Image chunk (e, R / 128, K stage)
// at ((e * MT + R / 128) * KC + stage) * kNvAChunk; g[e * N + R].
__global__ void nvfp4_weights_kernel(const uint8_t* codes, const uint16_t* scales, int E, int K, int N, int gate_up,
                                     int I, uint8_t* img, float* g_out)
{
    const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= (long long)E * N) return;
    const int e = (int)(t / N), R = (int)(t - (long long)e * N);
    const int n = gate_up ? nv_gate_up_column(R, I) : R;
    const uint8_t* c0 = codes + (size_t)e * (K / 2) * N + n;
    const uint16_t* s0 = scales + (size_t)e * (K / 32) * N + n;
    auto wval = [&](int k) {
        const uint32_t byte = c0[(size_t)(k >> 1) * N];
        return e2m1_value((k & 1) ? (byte >> 4) : (byte & 15u)) * bf16_bits_to_f32(s0[(size_t)(k >> 5) * N]);
    };
    float amax = 0.0f;
    for (int k = 0; k < K; ++k) amax = fmaxf(amax, fabsf(wval(k)));
    float g, d6;
    nv_row_scale(amax, g, d6);
    const int MT = N / kNvM, KC = K / kNvKc, r = R % kNvM;
    for (int b = 0; b < K / 16; ++b) {
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = wval(16 * b + i);
        uint32_t c[2];
        const uint32_t sb = nv_encode_block(v, g, d6, c);
        const int kc = b / 16, j = b % 16;
        uint8_t* chunk = img + (((size_t)e * MT + R / kNvM) * KC + kc) * kNvAChunk;
        *reinterpret_cast<uint2*>(chunk + nv_code_off(r, 8 * j)) = make_uint2(c[0], c[1]);
        chunk[nv_sfa_off(r, j)] = (uint8_t)sb;
    }
    g_out[t] = g;
}

// ---- token images (every forward) --------------------------------------------------
// Rows past a tile's count are written as zeros; slots past the tile count are
// left alone (no CTA reads them).  Image chunk (slot, stage) at (slot * KC +
// stage) * kNvBChunk; row scale gb[slot][n].

// gate_up: one warp per (tile slot, row n < 256) copies the encoded row of the
// token of sorted position pos0 + n (codes [T][K/2], scale factors [T][K/16],
// row scales [T], from nvfp4_rows_kernel) into the slot's image.
__global__ void nvfp4_gather_rows_kernel(const uint8_t* codes, const uint8_t* sf, const float* g, int K,
                                         const int32_t* tiles, const int32_t* n_tiles, const int32_t* sorted_pair,
                                         int top_k, uint8_t* img, float* gb)
{
    const long long wid = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int slot = (int)(wid / kNvN), n = (int)(wid % kNvN);
    if (slot >= *n_tiles) return;
    const int pos0 = tiles[3 * slot + 1], rows = tiles[3 * slot + 2];
    uint8_t* base = img + (size_t)slot * (K / kNvKc) * kNvBChunk;
    const bool live = n < rows;
    const int t = live ? sorted_pair[pos0 + n] / top_k : 0;
    const uint4* src = reinterpret_cast<const uint4*>(codes + (size_t)t * (K / 2));
    for (int c = lane; c < K / 32; c += 32) {   // 16-byte chunks: 8 per stage
        const uint4 v = live ? src[c] : make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(base + (size_t)(c >> 3) * kNvBChunk + nv_code_off(n, 16 * (c & 7))) = v;
    }
    const uint32_t* ssrc = reinterpret_cast<const uint32_t*>(sf + (size_t)t * (K / 16));
    for (int w = lane; w < K / 64; w += 32) {   // one word per k-block: 4 per stage
        const uint32_t v = live ? ssrc[w] : 0u;
        *reinterpret_cast<uint32_t*>(base + (size_t)(w >> 2) * kNvBChunk + nv_sfb_off(n, 4 * (w & 3))) = v;
    }
    if (lane == 0) gb[(size_t)slot * kNvN + n] = live ? g[t] : 0.0f;
}

// down: one warp per (tile slot, row n < 256) encodes act row pos0 + n (bf16,
// rows by sorted position) straight into the slot's image.
__global__ void nvfp4_token_rows_kernel(const uint16_t* src, int K, const int32_t* tiles, const int32_t* n_tiles,
                                        uint8_t* img, float* gb)
{
    const long long wid = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int slot = (int)(wid / kNvN), n = (int)(wid % kNvN);
    const int KC = K / kNvKc;
    if (slot >= *n_tiles) return;
    const int pos0 = tiles[3 * slot + 1], rows = tiles[3 * slot + 2];
    uint8_t* base = img + (size_t)slot * KC * kNvBChunk;
    if (n >= rows) {
        for (int b = lane; b < K / 16; b += 32) {
            uint8_t* chunk = base + (size_t)(b / 16) * kNvBChunk;
            *reinterpret_cast<uint2*>(chunk + nv_code_off(n, 8 * (b % 16))) = make_uint2(0u, 0u);
            chunk[nv_sfb_off(n, b % 16)] = 0;
        }
        if (lane == 0) gb[(size_t)slot * kNvN + n] = 0.0f;
        return;
    }
    const uint16_t* row = src + (size_t)(pos0 + n) * K;
    float amax = 0.0f;
    for (int b = lane; b < K / 16; b += 32) {
        float v[16];
        bf16x16_to_f32(row + 16 * b, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    float g, d6;
    nv_row_scale(amax, g, d6);
    for (int b = lane; b < K / 16; b += 32) {
        float v[16];
        bf16x16_to_f32(row + 16 * b, v);
        uint32_t c[2];
        const uint32_t sb = nv_encode_block(v, g, d6, c);
        uint8_t* chunk = base + (size_t)(b / 16) * kNvBChunk;
        *reinterpret_cast<uint2*>(chunk + nv_code_off(n, 8 * (b % 16))) = make_uint2(c[0], c[1]);
        chunk[nv_sfb_off(n, b % 16)] = (uint8_t)sb;
    }
    if (lane == 0) gb[(size_t)slot * kNvN + n] = g;
}

// ---- the block-scaled GEMM tile ----------------------------------------------------

struct NvParams {
    const uint8_t* a_img;     // [E][MT][KC] chunks of kNvAChunk bytes
    const float* a_g;         // [E][MT * 128] row scales
    int MT, KC;               // weight tiles per expert, K stages
    const uint8_t* b_img;     // [slots][KC] chunks of kNvBChunk bytes
    const float* b_g;         // [slots][256]
    const int32_t* tiles;     // [slots][3]: expert, first sorted position, rows (<= 256)
    const int32_t* n_tiles;
    uint16_t* out;            // bf16 rows by sorted position: act [P][I] (gate_up) or o [P][H] (down)
    int out_ld;
    uint32_t* status;
    unsigned long long timeout_ns;
};

// Matrix descriptor of a 32-row x 16-byte block of scale factors (no swizzle:
// 8-row core matrices 128 bytes apart), the source of tcgen05.cp 32x128b.
FE_DEV uint64_t nv_sf_desc(uint32_t saddr)
{
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)(128u >> 4) << 32;   // stride byte offset: 8-row core matrices
    d |= (uint64_t)1u << 46;            // descriptor version of tcgen05
    return d;                           // layout type 0: no swizzle
}

// Instruction descriptor of kind::mxf4nvf4: E2M1 A and B (format 1), both
// K-major, E4M3 scale factors (scale format 0), M = 128, N, dense K = 64.
__host__ __device__ constexpr uint32_t nv_instr_desc(int N)
{
    return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(kNvM >> 4) << 24);
}

// Copy a 32 x 128-bit block of scale factors into TMEM lanes 0..31 of 4
// consecutive columns, replicated to the other three lane quarters.
FE_DEV void nv_cp_sf(uint32_t taddr, uint64_t sdesc)
{
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

FE_DEV void nv_mma(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t tsfa, uint32_t tsfb,
                   uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb));
}

// grid: (weight tiles of one expert, tile slots); block: 4 warps.  Warp 0 lane 0
// loads stage i of A and B with one bulk copy each once the MMAs of stage i - 4
// are done; warp 1 (TMEM owner) lane 0 copies the stage's scale factors into
// TMEM and issues its 4 MMAs; after the K loop all 4 warps read the accumulator
// (TMEM lane quarter = warp) and write bf16 rows: gate_up SiLU(gate) * up into
// act, down into o for the ordered combine.
template <bool GATE_UP>
__global__ void __launch_bounds__(kNvThreads, 1) nvfp4_gemm_kernel(NvParams p)
{
    extern __shared__ uint8_t nv_dyn[];
    if ((int)blockIdx.y >= *p.n_tiles) return;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int slot = blockIdx.y, mt = blockIdx.x;
    const int e = p.tiles[3 * slot], pos0 = p.tiles[3 * slot + 1], rows = p.tiles[3 * slot + 2];
    const int nb = (rows + 15) & ~15;
    const int KC = p.KC;

    const uint32_t base0 = tc_saddr(nv_dyn);
    const uint32_t pad = (1024u - (base0 & 1023u)) & 1023u;
    uint8_t* sm = nv_dyn + pad;
    const uint32_t a_addr = tc_saddr(sm), b_addr = a_addr + kNvStages * kNvAChunk;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kNvStages * (kNvAChunk + kNvBChunk));
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kNvStages + 1);
    volatile int* flags = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const uint32_t bar0 = tc_saddr(bars);
    auto full = [&](int s) { return bar0 + 8u * (uint32_t)s; };
    auto empty = [&](int s) { return bar0 + 8u * (uint32_t)(kNvStages + s); };
    const uint32_t accf = bar0 + 8u * (uint32_t)(2 * kNvStages);

    if (tid == 0) {
        for (int s = 0; s < kNvStages; ++s) {
            tc_mbar_init(full(s), 1);
            tc_mbar_init(empty(s), 1);
        }
        tc_mbar_init(accf, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        flags[0] = 0;
    }
    if (warp == 1) {
        tc_alloc(tc_saddr(tmem_slot), kNvTmemCols);
        tc_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint8_t* a_src = p.a_img + ((size_t)e * p.MT + mt) * KC * kNvAChunk;
    const uint8_t* b_src = p.b_img + (size_t)slot * KC * kNvBChunk;

    if (warp == 0) {
        // ---- producer: one bulk copy per operand and stage ---------------------------------
        if (lane == 0) {
            int issued = 0;
            for (int i = 0; i < KC; ++i) {
                const int s = i % kNvStages;
                if (i >= kNvStages && !tc_mbar_wait(empty(s), ((i / kNvStages) - 1) & 1, p.timeout_ns)) flags[0] = 1;
                if (flags[0]) break;
                mbar_expect_tx(full(s), kNvAChunk + kNvBChunk);
                bulk_g2s(a_addr + s * kNvAChunk, a_src + (size_t)i * kNvAChunk, kNvAChunk, full(s));
                bulk_g2s(b_addr + s * kNvBChunk, b_src + (size_t)i * kNvBChunk, kNvBChunk, full(s));
                issued = i + 1;
            }
            // no copy outlives the CTA: wait (bounded) for the stages still in flight
            for (int i = max(0, issued - kNvStages); i < issued; ++i)
                if (!tc_mbar_wait(full(i % kNvStages), (i / kNvStages) & 1, p.timeout_ns)) flags[0] = 1;
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---- scale factors into TMEM, then the MMAs ------------------------------------------
        const uint32_t idesc = nv_instr_desc(nb);
        int issued = -1;
        for (int i = 0; i < KC; ++i) {
            const int s = i % kNvStages;
            if (!tc_mbar_wait(full(s), (i / kNvStages) & 1, p.timeout_ns)) flags[0] = 1;
            if (flags[0]) break;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t aa = a_addr + s * kNvAChunk, ba = b_addr + s * kNvBChunk;
                const uint32_t sfa = tmem + 256u + kNvSfCols * (uint32_t)s, sfb = sfa + 16u;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    nv_cp_sf(sfa + 4u * q, nv_sf_desc(aa + kNvACodes + 512u * q));
                    nv_cp_sf(sfb + 8u * q, nv_sf_desc(ba + kNvBCodes + 1024u * q));
                    nv_cp_sf(sfb + 8u * q + 4u, nv_sf_desc(ba + kNvBCodes + 1024u * q + 512u));
                }
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    nv_mma(tmem, tc_smem_desc(aa + 32u * q), tc_smem_desc(ba + 32u * q), idesc, sfa + 4u * q,
                           sfb + 8u * q, (i > 0 || q > 0) ? 1u : 0u);
                tc_commit(empty(s));
            }
            __syncwarp();
            issued = i;
        }
        if (lane == 0 && issued >= 0) tc_commit(accf);
        __syncwarp();
        if (issued >= 0 && !tc_mbar_wait(accf, 0, p.timeout_ns)) flags[0] = 1;
        if (issued < KC - 1) flags[0] = 1;
    }
    __syncthreads();

    // ---- epilogue: TMEM -> registers -> bf16 rows -----------------------------------------
    if (flags[0] != 0) {
        if (tid == 0) atomicOr(p.status, kDevTcTimeout);
    } else {
        tc_fence_after();
        const int row = 32 * warp + lane;   // A row of this thread's TMEM lane
        const float ga = p.a_g[(size_t)e * p.MT * kNvM + (size_t)mt * kNvM + row];
        const float* gb = p.b_g + (size_t)slot * kNvN;
        const uint32_t ta = tmem + ((uint32_t)(32 * warp) << 16);
#pragma unroll 1
        for (int c0 = 0; c0 < nb; c0 += 32) {
            uint32_t r[32];
            tc_ld16(ta + c0, *reinterpret_cast<uint32_t(*)[16]>(&r[0]));
            tc_ld16(ta + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&r[16]));
            tc_wait_ld();
            if (GATE_UP) {
                // lanes l and l + 16 hold gate and up of one act column: the gate lane
                // takes tokens c0 .. c0 + 15, the up lane tokens c0 + 16 .. c0 + 31
                const bool up = lane & 16;
                const int acol = 64 * mt + 16 * warp + (lane & 15);
#pragma unroll
                for (int n = 0; n < 16; ++n) {
                    const float lo = __uint_as_float(r[n]) * ga, hi = __uint_as_float(r[16 + n]) * ga;
                    const float other = __shfl_xor_sync(0xffffffffu, up ? lo : hi, 16);
                    const int tn = up ? 16 + n : n;
                    const float own = up ? hi : lo;
                    const float gv = (up ? other : own) * gb[c0 + tn], uv = (up ? own : other) * gb[c0 + tn];
                    if (c0 + tn < rows) {
                        const float a = silu_mul(gv, uv);
                        const __nv_bfloat16 v = __float2bfloat16_rn(a);
                        p.out[(size_t)(pos0 + c0 + tn) * p.out_ld + acol] = *reinterpret_cast<const uint16_t*>(&v);
                    }
                }
            } else {
                const int col = kNvM * mt + row;
#pragma unroll
                for (int n = 0; n < 32; ++n)
                    if (c0 + n < rows) {
                        const __nv_bfloat16 v = __float2bfloat16_rn(__uint_as_float(r[n]) * ga * gb[c0 + n]);
                        p.out[(size_t)(pos0 + c0 + n) * p.out_ld + col] = *reinterpret_cast<const uint16_t*>(&v);
                    }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tc_dealloc(tmem, kNvTmemCols);
}

}  // namespace fe
