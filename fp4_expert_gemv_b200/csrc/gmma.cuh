// Grouped FP4 projection for any number of tokens: one CTA per (routed
// expert, unit), all the expert's tokens as the N dimension of tensor-core
// mma.m16n8k16 in blocks of 8.
//
// "FireEcho Engine", section "The Goliath Kernel: Why It's Fast" (packed
// bytes loaded, nibbles dequantised in registers, tensor-core accumulation,
// expert IDs read from device memory) and "Speed Optimization History"
// (grouped dispatch, fused gate_up, one launch for all routed experts).
//
// A gate_up unit is 16 gate columns and the 16 up columns of the same act
// outputs (two fragment-ordered blocks, contiguous), a down unit is 16 output
// columns (one block).  The CTA fetches its unit with one TMA bulk copy,
// stages the B rows of 8 tokens at a time (x rows for gate_up, act rows for
// down, as fp16 pairs with a per-row power-of-two shift), lets each of its 8
// warps run the mma over a strided set of 64-k quads, and reduces the warps'
// partial sums in shared memory; gate_up applies SiLU(gate)*up before writing
// act (fp32, by grouped pair position), down writes o (fp32, by position).
#pragma once

#include "common.cuh"
#include "mma.cuh"

namespace fe {

constexpr int kGmmaThreads = 256;
constexpr int kGmmaWarps = kGmmaThreads / 32;

struct GmmaParams {
    const uint8_t* blocks;    // gate_up: [E][I/16] units of 2 blocks; down: [E][H/16] blocks
    int K;                    // reduction length (H for gate_up, I for down)
    int n_units;              // units per expert
    int N_out;                // row length of out (I for gate_up, H for down)
    const int32_t* offsets;   // [E+1]
    const int32_t* active;    // [E]
    const int32_t* n_active;  // [1]
    const int32_t* sorted_pair;
    int top_k;
    const uint16_t* x;        // gate_up B source: bf16 [T][H]
    const float* act_in;      // down B source: fp32 [P][I] by position
    float* out;               // act [P][I] or o [P][H] by position
    uint32_t* status;
    unsigned long long timeout_ns;
};

__host__ __device__ inline uint32_t gmma_unit_bytes(bool gate_up, int K) { return (gate_up ? 2u : 1u) * block_bytes(K); }

// Dynamic shared memory: [unit bytes][mbarrier 16][B rows 9 x brow_words(K)][shift 8][red 8 x 32 x 8 floats]
__host__ __device__ inline size_t gmma_smem_bytes(bool gate_up, int K)
{
    return (size_t)gmma_unit_bytes(gate_up, K) + 16 + 4u * 9 * brow_words(K) + 4 * 8 + 4 * kGmmaWarps * 32 * 8;
}

FE_DEV uint32_t gsmem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

template <bool GATE_UP>
__global__ void __launch_bounds__(kGmmaThreads) gmma_kernel(GmmaParams p)
{
    extern __shared__ __align__(128) uint8_t gs[];
    const int a = blockIdx.x / p.n_units;
    const int unit = blockIdx.x - a * p.n_units;
    if (a >= *p.n_active) return;
    const int e = p.active[a];
    const int pos0 = p.offsets[e], npos = p.offsets[e + 1] - pos0;
    const int K = p.K;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t = lane & 3;
    const uint32_t ubytes = gmma_unit_bytes(GATE_UP, K);
    const int rw = brow_words(K);

    uint8_t* ubuf = gs;
    uint64_t* bar = reinterpret_cast<uint64_t*>(gs + ubytes);
    uint32_t* rows = reinterpret_cast<uint32_t*>(gs + ubytes + 16);
    int* shift = reinterpret_cast<int*>(rows + 9 * rw);
    float* red = reinterpret_cast<float*>(shift + 8);

    const uint32_t b = gsmem_addr(bar);
    if (tid == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(b) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    for (int i = tid; i < rw; i += kGmmaThreads) rows[8 * rw + i] = 0u;   // the zero row
    __syncthreads();
    if (tid == 0) {
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(b), "r"(ubytes) : "memory");
        asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                         gsmem_addr(ubuf)),
                     "l"(p.blocks + ((size_t)e * p.n_units + unit) * ubytes), "r"(ubytes), "r"(b)
                     : "memory");
    }
    bool loaded = false;

    for (int nb = 0; nb * 8 < npos; ++nb) {
        const int nvalid = min(8, npos - 8 * nb);
        // stage the B rows of this n-block: warp w -> row w
        if (warp < nvalid) {
            const int pos = pos0 + 8 * nb + warp;
            int s;
            if (GATE_UP) {
                const int tok = p.sorted_pair[pos] / p.top_k;
                s = warp_stage_row<true>(p.x + (size_t)tok * K, K, rows + warp * rw, lane);
            } else {
                s = warp_stage_row<false>(p.act_in + (size_t)pos * K, K, rows + warp * rw, lane);
            }
            if (lane == 0) shift[warp] = s;
        }
        if (!loaded) {
            // bounded wait for the unit's bytes (all threads)
            bool ok = false;
            const unsigned long long t0 = globaltimer_ns();
            while (!ok) {
                uint32_t r;
                asm volatile(
                    "{\n\t.reg .pred q;\n\tmbarrier.try_wait.parity.shared::cta.b64 q, [%1], 0;\n\tselp.u32 %0, 1, 0, q;\n\t}"
                    : "=r"(r)
                    : "r"(b)
                    : "memory");
                ok = r != 0;
                if (!ok && globaltimer_ns() - t0 > p.timeout_ns) break;
            }
            if (!ok) {
                if (tid == 0) atomicOr(p.status, 0x8u);
                return;   // timed out: the copy is not coming
            }
            loaded = true;
        }
        __syncthreads();
        const uint32_t* brow = rows + (g < nvalid ? g : 8) * rw;
        float t0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, t1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        for (int q = warp; q < K / 64; q += kGmmaWarps) {
            if (GATE_UP)
                quad_mma2(ubuf, ubuf + block_bytes(K), K, brow, q, lane, t0, t1);
            else
                quad_mma(ubuf, K, brow, q, lane, t0);
        }
        float* rl = red + (warp * 32 + lane) * 8;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            rl[i] = t0[i];
            rl[4 + i] = t1[i];
        }
        __syncthreads();
        if (tid < 128) {
            const int n = tid & 15, j = tid >> 4;   // output column, token of the n-block
            if (j < nvalid) {
                const int ln = 4 * (n & 7) + (j >> 1), idx = (n >> 3) * 2 + (j & 1);
                float s0 = 0.0f, s1 = 0.0f;
#pragma unroll
                for (int w = 0; w < kGmmaWarps; ++w) {
                    s0 += red[(w * 32 + ln) * 8 + idx];
                    s1 += red[(w * 32 + ln) * 8 + 4 + idx];
                }
                const float m = pow2f(shift[j]);
                const int pos = pos0 + 8 * nb + j;
                p.out[(size_t)pos * p.N_out + 16 * unit + n] = GATE_UP ? silu_mul(s0 * m, s1 * m) : s0 * m;
            }
        }
        __syncthreads();
    }
    (void)t;
}

}  // namespace fe
