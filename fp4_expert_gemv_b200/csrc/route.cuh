// Router (top-k + softmax over the selected logits) and expert grouping
// (histogram, exclusive scan, stable scatter) in one single-CTA kernel.
//
// "FireEcho Engine", sections "Speed Optimization History" (step 1, grouped
// dispatch; step 5, packed MoE) and "The Goliath Kernel: Why It's Fast" (the
// kernel reads expert IDs from a GPU tensor, no host synchronisation): the
// routing and the per-expert pair lists are produced on the device and read
// by the projection kernels from device memory.
#pragma once

#include "common.cuh"
#include "stream.cuh"   // SgSplit, sg_plan_ranges

namespace fe {

struct RouteParams {
    const float* logits;   // [T][E]
    int T, E, k;
    int32_t* idx;          // [T][k]   experts, descending logit
    float* w;              // [T][k]   softmax of the selected logits
    int32_t* counts;       // [E]
    int32_t* offsets;      // [E+1]    exclusive scan of counts
    int32_t* sorted_pair;  // [T*k]    pair ids ordered by (expert, pair id)
    int32_t* pair_row;     // [T*k]    inverse of sorted_pair
    int32_t* active;       // [E]      experts with count > 0, ascending
    int32_t* n_active;     // [1]
    int32_t* max_count;    // [1]      largest per-expert count
    uint32_t* status;
    SgSplit split;         // work split of the streaming kernels, filled when split.table is set
};

// (value, index) order of the router: larger logit first, equal logits by
// lower expert index.  NaN has been mapped to -inf before this is used.
FE_DEV bool route_better(float va, int ia, float vb, int ib)
{
    return (va > vb) || (va == vb && ia < ib);
}

constexpr int kRouteMaxPerLane = 32;  // E <= 1024

constexpr int kRouteMaxThreads = 512;

// Dynamic shared memory: cnt[E] | cursor[E] | wcnt[nwarps][E]
__host__ __device__ inline int route_plan_offset(int E, int nthreads);

__global__ void __launch_bounds__(kRouteMaxThreads) route_group_kernel(RouteParams p)
{
    extern __shared__ int32_t sm[];
    const int E = p.E, k = p.k, T = p.T;
    const int nthreads = blockDim.x, nwarps = nthreads >> 5;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int32_t* cnt = sm;
    int32_t* cursor = sm + E;
    int32_t* wcnt = sm + 2 * E;

    // ---- router: one warp per token --------------------------------------
    for (int t = warp; t < T; t += nwarps) {
        const float* row = p.logits + (size_t)t * E;
        float v[kRouteMaxPerLane];
        bool nan_seen = false;
#pragma unroll
        for (int i = 0; i < kRouteMaxPerLane; ++i) {
            const int e = lane + 32 * i;
            float x = (e < E) ? row[e] : -INFINITY;
            if (x != x) { nan_seen = true; x = -INFINITY; }
            v[i] = x;
        }
        if (__any_sync(0xffffffffu, nan_seen) && lane == 0) atomicOr(p.status, kDevNanLogit);
        uint32_t taken = 0;
        for (int j = 0; j < k; ++j) {
            float bv = -INFINITY;
            int bi = 0x7fffffff;
#pragma unroll
            for (int i = 0; i < kRouteMaxPerLane; ++i) {
                const int e = lane + 32 * i;
                if (e < E && !((taken >> i) & 1u) && route_better(v[i], e, bv, bi)) { bv = v[i]; bi = e; }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                if (route_better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
            }
            if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
            if (lane == 0) {
                p.idx[(size_t)t * k + j] = bi;
                p.w[(size_t)t * k + j] = bv;   // the logit for now
            }
        }
        __syncwarp();
        // softmax over the k selected logits
        const float l0 = p.w[(size_t)t * k];
        float s = 0.0f;
        for (int j = lane; j < k; j += 32) s += expf(p.w[(size_t)t * k + j] - l0);
        s = warp_sum(s);
        __syncwarp();
        for (int j = lane; j < k; j += 32) {
            const float ej = expf(p.w[(size_t)t * k + j] - l0);
            p.w[(size_t)t * k + j] = ej / s;
        }
    }
    __syncthreads();

    // ---- grouping ---------------------------------------------------------
    const int P = T * k;
    for (int e = tid; e < E; e += nthreads) cnt[e] = 0;
    __syncthreads();
    for (int q = tid; q < P; q += nthreads) {
        const int e = p.idx[q];
        if (e < 0 || e >= E) { atomicOr(p.status, kDevBadExpert); continue; }
        atomicAdd(&cnt[e], 1);
    }
    __syncthreads();
    if (warp == 0) {
        // exclusive scan of the counts and of the "has pairs" flags by one warp
        const int per = (E + 31) / 32;
        const int e0 = lane * per;
        int sum = 0, nact = 0, mx = 0;
        for (int e = e0; e < e0 + per && e < E; ++e) {
            sum += cnt[e];
            nact += cnt[e] > 0;
            mx = max(mx, cnt[e]);
        }
        int incl = sum, inact = nact;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int a = __shfl_up_sync(0xffffffffu, incl, o);
            const int b = __shfl_up_sync(0xffffffffu, inact, o);
            if (lane >= o) { incl += a; inact += b; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        int run = incl - sum, arun = inact - nact;
        for (int e = e0; e < e0 + per && e < E; ++e) {
            const int c = cnt[e];
            p.counts[e] = c;
            p.offsets[e] = run;
            cursor[e] = run;
            if (c > 0) p.active[arun++] = e;
            run += c;
        }
        if (lane == 31) {
            p.offsets[E] = incl;
            *p.n_active = inact;
            *p.max_count = mx;
        }
    }
    __syncthreads();
    if (p.split.table) {
        long long* scratch = reinterpret_cast<long long*>(sm + route_plan_offset(E, nthreads));
        sg_plan_ranges(p.split, p.counts, p.active, *p.n_active, scratch);
    }

    // stable scatter, one chunk of nthreads pairs at a time: the position of a
    // pair is its expert's cursor + pairs of that expert in earlier warps of the
    // chunk + pairs of that expert in earlier lanes of its warp.
    const uint32_t lt_mask = (1u << lane) - 1u;
    for (int base = 0; base < P; base += nthreads) {
        const int q = base + tid;
        int e = (q < P) ? p.idx[q] : -1;
        if (e >= E) e = -1;
        for (int i = tid; i < nwarps * E; i += nthreads) wcnt[i] = 0;
        __syncthreads();
        const uint32_t peers = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(peers & lt_mask);
        if (e >= 0 && rank == 0) wcnt[warp * E + e] = __popc(peers);
        __syncthreads();
        for (int ee = tid; ee < E; ee += nthreads) {
            int run = cursor[ee];
            for (int w2 = 0; w2 < nwarps; ++w2) {
                const int c = wcnt[w2 * E + ee];
                wcnt[w2 * E + ee] = run;
                run += c;
            }
            cursor[ee] = run;
        }
        __syncthreads();
        if (e >= 0) {
            const int pos = wcnt[warp * E + e] + rank;
            p.sorted_pair[pos] = q;
            p.pair_row[q] = pos;
        }
        __syncthreads();
    }
}

// Shared memory of route_group_kernel: counts, cursors, per-warp counts, then
// (8-byte aligned) the scratch of the streaming kernels' work split.
__host__ __device__ inline int route_plan_offset(int E, int nthreads) { return (E * (2 + nthreads / 32) + 1) & ~1; }
inline size_t route_smem_bytes(int E, int nthreads)
{
    return sizeof(int32_t) * (size_t)route_plan_offset(E, nthreads) + sizeof(long long) * (2 * ((size_t)E + 1) + 32);
}

}  // namespace fe
