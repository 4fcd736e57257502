// Router and expert grouping for many tokens, spread over the whole GPU.
//
// "FireEcho Engine", sections "Speed Optimization History" (grouped
// dispatch) and "The Goliath Kernel: Why It's Fast" (expert ids stay on the
// device).  The single-CTA route_group_kernel serialises thousands of tokens;
// here the same outputs come from four launches:
//
//   1. route_tokens_kernel: one warp per token selects the top-k logits
//      (warp_route: lane maxima threshold, candidates ranked by counting) and
//      takes the softmax over them -> idx, w;
//   2. group_hist_kernel: block b counts the experts of its kGroupChunk pairs;
//   3. group_scan_kernel: counts, exclusive offsets, and for every (expert,
//      block) the first sorted position of that block's pairs of the expert;
//      also the active-expert list and the largest count;
//   4. group_scatter_kernel: block b places its pairs: position = its block
//      base + pairs of the same expert earlier in the block (warp match, then
//      a running count per expert across the block's chunks), so the order by
//      (expert, pair id) is the stable one, with no atomics deciding an order.
#pragma once

#include "common.cuh"
#include "warp_route.cuh"
#include "route.cuh"    // RouteParams

namespace fe {

constexpr int kRouteWarps = 8;       // tokens per block in route_tokens_kernel
constexpr int kRouteCand = 256;      // candidate keys per routing warp: >= max(64, k * E/32) for k <= 16, E <= 512
constexpr int kGroupChunk = 2048;    // pairs per grouping block
constexpr int kGroupThreads = 256;

// Routing for many tokens applies when one warp can route a token.
__host__ __device__ inline bool route_large_ok(int E, int k) { return E <= kDecMaxE && k <= 16; }

__global__ void __launch_bounds__(kRouteWarps * 32) route_tokens_kernel(RouteParams p)
{
    __shared__ unsigned long long cand[kRouteWarps][kRouteCand];
    __shared__ int sel_e[kRouteWarps][16];
    __shared__ float sel_w[kRouteWarps][16];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * kRouteWarps + warp;
    if (t >= p.T) return;
    const int k = p.k;
    const bool nan = warp_route(p.logits + (size_t)t * p.E, p.E, k, lane, cand[warp], kRouteCand, sel_e[warp], sel_w[warp]);
    if (nan && lane == 0) atomicOr(p.status, kDevNanLogit);
    __syncwarp();
    warp_softmax(sel_w[warp], k, lane);
    if (lane < k) {
        p.idx[(size_t)t * k + lane] = sel_e[warp][lane];
        p.w[(size_t)t * k + lane] = sel_w[warp][lane];
    }
}

// bh: [nblocks][E] pair counts per block and expert.
__global__ void __launch_bounds__(kGroupThreads) group_hist_kernel(const int32_t* idx, int P, int E, int32_t* bh)
{
    extern __shared__ int32_t grp_hist_sm[];
    int32_t* hist = grp_hist_sm;
    for (int e = threadIdx.x; e < E; e += kGroupThreads) hist[e] = 0;
    __syncthreads();
    const int p0 = blockIdx.x * kGroupChunk, p1 = min(P, p0 + kGroupChunk);
    for (int q = p0 + threadIdx.x; q < p1; q += kGroupThreads) {
        const int e = idx[q];
        if (e >= 0 && e < E) atomicAdd(&hist[e], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kGroupThreads) bh[(size_t)blockIdx.x * E + e] = hist[e];
}

// One block: counts, offsets, per-(block, expert) bases (in place in bh),
// active list, n_active, max_count.  Thread e walks the blocks of expert e.
__global__ void __launch_bounds__(1024) group_scan_kernel(int32_t* bh, int nblocks, int E, int32_t* counts,
                                                          int32_t* offsets, int32_t* active, int32_t* n_active,
                                                          int32_t* max_count, SgSplit split)
{
    extern __shared__ int32_t grp_scan_sm[];   // [E] counts, then [E] scan
    __shared__ int wsum[32], wact[32], wmx[32];
    int32_t* sc = grp_scan_sm;
    const int nthreads = blockDim.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (E + nthreads - 1) / nthreads, e0 = tid * per;
    // each thread: the counts of a contiguous run of experts
    int loc = 0, lact = 0, lmx = 0;
    for (int e = e0; e < e0 + per && e < E; ++e) {
        int c = 0;
        for (int b = 0; b < nblocks; ++b) c += bh[(size_t)b * E + e];
        sc[e] = c;
        loc += c;
        lact += c > 0;
        lmx = max(lmx, c);
    }
    // block scans of the pair counts and of the active flags, and the largest count
    int incl = loc, iact = lact, mx = lmx;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int a = __shfl_up_sync(0xffffffffu, incl, o), c = __shfl_up_sync(0xffffffffu, iact, o);
        if (lane >= o) {
            incl += a;
            iact += c;
        }
        mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    if (lane == 31) {
        wsum[warp] = incl;
        wact[warp] = iact;
    }
    if (lane == 0) wmx[warp] = mx;
    __syncthreads();
    int base = 0, abase = 0, tmax = 0;
    for (int w = 0; w < nthreads / 32; ++w) {
        if (w < warp) {
            base += wsum[w];
            abase += wact[w];
        }
        tmax = max(tmax, wmx[w]);
    }
    int run = base + incl - loc, arun = abase + iact - lact;
    for (int e = e0; e < e0 + per && e < E; ++e) {
        const int c = sc[e];
        sc[E + e] = run;
        offsets[e] = run;
        counts[e] = c;
        if (c > 0) active[arun++] = e;
        run += c;
    }
    if (tid == nthreads - 1) {
        offsets[E] = base + incl;
        *n_active = abase + iact;
        *max_count = tmax;
    }
    __syncthreads();
    if (split.table) sg_plan_ranges(split, counts, active, *n_active, reinterpret_cast<long long*>(sc + 2 * ((E + 1) & ~1)));
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = sc[E + e];
        for (int b = 0; b < nblocks; ++b) {
            const int c = bh[(size_t)b * E + e];
            bh[(size_t)b * E + e] = run;
            run += c;
        }
    }
}

// Block b places pairs [b * kGroupChunk, ...) in chunks of kGroupThreads: a
// pair's position is its block base for the expert, plus the pairs of that
// expert in earlier chunks of the block (cnt), in earlier warps of this chunk
// (wc) and in earlier lanes of its warp (match mask).
__global__ void __launch_bounds__(kGroupThreads) group_scatter_kernel(const int32_t* idx, int P, int E,
                                                                      const int32_t* bh, int32_t* sorted_pair,
                                                                      int32_t* pair_row, uint32_t* status)
{
    extern __shared__ int32_t grp_scatter_sm[];   // cnt [E], wc [8][E]
    int32_t* gs = grp_scatter_sm;
    constexpr int W = kGroupThreads / 32;
    int32_t* cnt = gs;
    int32_t* wc = gs + E;
    for (int i = threadIdx.x; i < E * (W + 1); i += kGroupThreads) gs[i] = 0;
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t lt = (1u << lane) - 1u;
    const int p0 = blockIdx.x * kGroupChunk, p1 = min(P, p0 + kGroupChunk);
    for (int c0 = p0; c0 < p1; c0 += kGroupThreads) {
        const int q = c0 + threadIdx.x;
        int e = -1;
        if (q < p1) {
            e = idx[q];
            if (e < 0 || e >= E) {
                atomicOr(status, kDevBadExpert);
                e = -1;
            }
        }
        const uint32_t m = __match_any_sync(0xffffffffu, e);
        const bool leader = e >= 0 && (m & lt) == 0;
        if (leader) wc[warp * E + e] = __popc(m);
        __syncthreads();
        if (e >= 0) {
            int pre = cnt[e] + __popc(m & lt);
            for (int w2 = 0; w2 < warp; ++w2) pre += wc[w2 * E + e];
            const int pos = bh[(size_t)blockIdx.x * E + e] + pre;
            sorted_pair[pos] = q;
            pair_row[q] = pos;
        }
        __syncthreads();
        if (leader) {
            atomicAdd(&cnt[e], __popc(m));
            wc[warp * E + e] = 0;
        }
        __syncthreads();
    }
}

}  // namespace fe
