// Router GEMM fused with the top-k: logits = x W_r^T (x bf16 [T][H], W_r bf16
// [E][H], one row per expert, fp32 accumulation), then for every token the k
// largest logits and the softmax over them, in one launch.
//
// "FireEcho Engine", sections "Architecture" (MoEFFN: packed MoE whose dispatch
// starts from the router's scores) and "Speed Optimization History" (step 1:
// the router in front of the grouped dispatch; expert ids chosen on the GPU).
//
// One CTA per (16-token tile, 32 experts, K split): four warps, each a 16 x 8
// tensor-core tile (mma.m16n8k16, bf16 operands, fp32 accumulators) over its
// share of K.  A lane reads its x rows and its W_r row in 16-byte runs; within
// a 64-wide chunk of K, lane c of a quad holds physical k = 16c .. 16c+15 and
// feeds k 16c + 4s .. 16c + 4s + 3 to mma step s as the fragment's
// (2c, 2c+1, 2c+8, 2c+9).  A and B use the same map, so the sum over K is the
// same dot product.  Every CTA writes its fp32 partial; the last CTA of a token
// tile to finish (an atomic ticket, no waiting) adds the K splits in order,
// writes the logits and routes the tile's tokens (warp_route.cuh).  At small T
// the K splits spread W_r over more SMs: the layer's W_r is read once.
#pragma once

#include "common.cuh"
#include "warp_route.cuh"

namespace fe {

constexpr int kRtTok = 16;          // tokens per tile (the mma's M)
constexpr int kRtExp = 32;          // experts per CTA: 4 warps x 8 (the mma's N)
constexpr int kRtThreads = 128;
constexpr int kRtMaxSplits = 8;     // K splits at most
constexpr int kRtMaxK = 32;         // top_k at most (a lane per slot)
constexpr int kRtCand = 256;        // routing candidates per warp: k * ceil(E / 32) at most
constexpr int kRtSplitFloats = 32768;   // K-split partials kept when K is split (floats)

struct RouterParams {
    const uint16_t* x;     // [T][H] bf16
    const uint16_t* wr;    // [E][H] bf16
    int T, H, E, k, ks;    // ks: K splits (H / ks a multiple of 64)
    float* part;           // [ks][T][E] fp32 partials
    unsigned* ticket;      // [ceil(T / 16)]: CTAs of the tile done; the last one resets it
    float* logits;         // [T][E]
    int32_t* idx;          // [T][k] or null
    float* w;              // [T][k] or null
    uint32_t* status;
};

FE_DEV void mma16816_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                          uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The 8 words (16 bf16) of physical k = 16c .. 16c+15 of a row, or zeros.
FE_DEV void rt_load_run(const uint16_t* row, bool valid, uint32_t (&v)[8])
{
    if (valid) {
        const uint4 lo = __ldg(reinterpret_cast<const uint4*>(row));
        const uint4 hi = __ldg(reinterpret_cast<const uint4*>(row + 8));
        v[0] = lo.x; v[1] = lo.y; v[2] = lo.z; v[3] = lo.w;
        v[4] = hi.x; v[5] = hi.y; v[6] = hi.z; v[7] = hi.w;
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = 0u;
    }
}

__global__ void __launch_bounds__(kRtThreads) router_kernel(RouterParams p)
{
    __shared__ unsigned long long cand[kRtThreads / 32][kRtCand];
    __shared__ int sel_e[kRtThreads / 32][kRtMaxK];
    __shared__ float sel_w[kRtThreads / 32][kRtMaxK];
    __shared__ int last;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, c = lane & 3;
    const int T = p.T, H = p.H, E = p.E;
    const int t0 = blockIdx.x * kRtTok, e0 = blockIdx.y * kRtExp + warp * 8;
    const int hs = H / p.ks, k0 = blockIdx.z * hs;
    const int ta = t0 + g, tb = t0 + g + 8, ew = e0 + g;
    const bool va = ta < T, vb = tb < T, vw = ew < E;
    const uint16_t* xa = p.x + (size_t)(va ? ta : 0) * H + k0 + 16 * c;
    const uint16_t* xb = p.x + (size_t)(vb ? tb : 0) * H + k0 + 16 * c;
    const uint16_t* wrow = p.wr + (size_t)(vw ? ew : 0) * H + k0 + 16 * c;
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll 4
    for (int kc = 0; kc < hs; kc += 64) {
        uint32_t ra[8], rb[8], rw[8];
        rt_load_run(xa + kc, va, ra);
        rt_load_run(xb + kc, vb, rb);
        rt_load_run(wrow + kc, vw, rw);
#pragma unroll
        for (int s = 0; s < 4; ++s)
            mma16816_bf16(acc, ra[2 * s], rb[2 * s], ra[2 * s + 1], rb[2 * s + 1], rw[2 * s], rw[2 * s + 1]);
    }
    // accumulator: (token ta, experts e0 + 2c, + 1) and (token tb, the same experts)
    float* part = p.part + (size_t)blockIdx.z * T * E;
    const int ec = e0 + 2 * c;
    if (va) {
        if (ec < E) part[(size_t)ta * E + ec] = acc[0];
        if (ec + 1 < E) part[(size_t)ta * E + ec + 1] = acc[1];
    }
    if (vb) {
        if (ec < E) part[(size_t)tb * E + ec] = acc[2];
        if (ec + 1 < E) part[(size_t)tb * E + ec + 1] = acc[3];
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const unsigned n = gridDim.y * gridDim.z;
        last = atomicAdd(p.ticket + blockIdx.x, 1u) == n - 1u;
    }
    __syncthreads();
    if (!last) return;
    __threadfence();
    // the last CTA of the tile: the K splits added in order (every CTA of the tile has
    // written its partial), then the logits
    const int nt = min(kRtTok, T - t0);
    for (int i = tid; i < nt * E; i += kRtThreads) {
        const size_t o = (size_t)(t0 + i / E) * E + (i % E);
        float v[kRtMaxSplits];
#pragma unroll
        for (int q = 0; q < kRtMaxSplits; ++q) v[q] = q < p.ks ? __ldcg(p.part + (size_t)q * T * E + o) : 0.0f;
        float sum = v[0];
#pragma unroll
        for (int q = 1; q < kRtMaxSplits; ++q)
            if (q < p.ks) sum += v[q];
        p.logits[o] = sum;
    }
    __syncthreads();   // the tile's logits, for this CTA's warps
    for (int t = t0 + warp; t < t0 + nt; t += kRtThreads / 32) {
        const bool nan = warp_route(p.logits + (size_t)t * E, E, p.k, lane, cand[warp], kRtCand, sel_e[warp],
                                    sel_w[warp]);
        if (nan && lane == 0) atomicOr(p.status, kDevNanLogit);
        warp_softmax(sel_w[warp], p.k, lane);
        if (lane < p.k) {
            if (p.idx) p.idx[(size_t)t * p.k + lane] = sel_e[warp][lane];
            if (p.w) p.w[(size_t)t * p.k + lane] = sel_w[warp][lane];
        }
        __syncwarp();
    }
    if (tid == 0) p.ticket[blockIdx.x] = 0u;   // every CTA of the tile has arrived: ready for the next launch
}

// K splits for T tokens: enough CTAs to spread W_r when T is small, at most
// kRtMaxSplits, H / ks a multiple of 64, the partials within kRtSplitFloats.
__host__ inline int router_splits(int T, int H, int E)
{
    const long long tiles = (T + kRtTok - 1) / kRtTok, cpt = (E + kRtExp - 1) / kRtExp;
    int ks = 1;
    while (ks * 2 <= kRtMaxSplits && (H / 64) % (ks * 2) == 0 && tiles * cpt * ks * 2 <= 64 &&
           (long long)ks * 2 * T * E <= kRtSplitFloats)
        ks *= 2;
    return ks;
}

}  // namespace fe
