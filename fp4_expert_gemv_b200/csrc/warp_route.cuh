// Router of one token row by one warp: top-k by logit (ties to the lower
// expert index) and the softmax over the k selected logits.
//
// "FireEcho Engine", sections "Speed Optimization History" (step 1, grouped
// dispatch) and "The Goliath Kernel: Why It's Fast" (expert ids chosen and kept
// on the GPU).
#pragma once

#include "common.cuh"

namespace fe {

// ---- routing ---------------------------------------------------------------------
// Orderable key of logit v of expert e: a larger key ranks first.  NaN ranks
// as -inf, -0 as +0, and among equal logits the lower expert index ranks
// first, so keys are unique and the top-k order is the stable one.  A valid
// key is never 0.
FE_DEV unsigned long long route_key(float v, int e)
{
    uint32_t u = __float_as_uint(v != v ? -INFINITY : v);
    if ((u << 1) == 0u) u = 0u;
    const uint32_t ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ((unsigned long long)ord << 32) | (0xffffffffu - (uint32_t)e);
}

FE_DEV float route_key_value(unsigned long long key)
{
    const uint32_t ord = (uint32_t)(key >> 32);
    return __uint_as_float((ord & 0x80000000u) ? (ord & 0x7fffffffu) : ~ord);
}

FE_DEV int route_key_expert(unsigned long long key) { return (int)(0xffffffffu - (uint32_t)key); }

// One warp selects the top-k (E <= 32 J) logits of one token row (global
// memory), writing slot r = rank r: sel_e[r] expert, sel_w[r] logit.  Lane l
// holds the keys of experts l, l+32, ...  A threshold theta such that k
// lanes hold a key >= theta puts every key of the top k among the
// candidates (keys >= theta), and since every key above a candidate is a
// candidate too, a candidate's rank among the candidates is its rank among
// all E.  theta is first the k-th largest lane maximum by value (one 32-bit
// pass, ties counted); if that leaves more than 64 candidates (values tied
// around it) it is refined to the k-th largest lane maximum key, which
// leaves at most k J.  The candidates go to `cand` at slots counted from
// ballots and each is ranked by counting.  cap >= max(64, k J) is the caller's
// guarantee.  Returns whether the row holds a NaN (warp-uniform).
template <int J>
FE_DEV bool warp_topk(const float* row, int E, int k, int lane, unsigned long long* cand, int cap, int* sel_e,
                      float* sel_w)
{
    constexpr unsigned FULL = 0xffffffffu;
    unsigned long long key[J];
    unsigned long long kmax = 0ull;
    bool nan = false;
#pragma unroll
    for (int j = 0; j < J; ++j) {
        const int e = lane + 32 * j;
        key[j] = 0ull;
        if (e < E) {
            const float v = row[e];
            nan |= v != v;
            key[j] = route_key(v, e);
        }
        kmax = kmax > key[j] ? kmax : key[j];
    }
    // a lane whose maximum is below the k-th largest has >= k lanes strictly
    // above it; lanes without a logit (E < 32) hold 0, below every valid key
    const uint32_t omax = (uint32_t)(kmax >> 32);
    int r0 = 0, r1 = 0, r2 = 0, r3 = 0;
#pragma unroll
    for (int s = 0; s < 32; s += 4) {
        r0 += __shfl_sync(FULL, omax, s) > omax;
        r1 += __shfl_sync(FULL, omax, s + 1) > omax;
        r2 += __shfl_sync(FULL, omax, s + 2) > omax;
        r3 += __shfl_sync(FULL, omax, s + 3) > omax;
    }
    const uint32_t theta = __reduce_min_sync(FULL, (r0 + r1 + r2 + r3) < k ? omax : 0xffffffffu);
    const unsigned long long theta_key = (unsigned long long)theta << 32;   // smallest key of value theta
    int nc = 0;
#pragma unroll
    for (int j = 0; j < J; ++j) nc += __popc(__ballot_sync(FULL, key[j] >= theta_key));
    unsigned long long th = theta_key;
    if (nc > 64) {
        int q0 = 0, q1 = 0;
#pragma unroll
        for (int s = 0; s < 32; s += 2) {
            q0 += __shfl_sync(FULL, kmax, s) > kmax;
            q1 += __shfl_sync(FULL, kmax, s + 1) > kmax;
        }
        unsigned long long m = (q0 + q1) < k ? kmax : ~0ull;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const unsigned long long other = __shfl_xor_sync(FULL, m, o);
            m = other < m ? other : m;
        }
        th = m;
    }
    const uint32_t lt = (1u << lane) - 1u;
    nc = 0;
#pragma unroll
    for (int j = 0; j < J; ++j) {
        const bool c = key[j] >= th;
        const uint32_t bj = __ballot_sync(FULL, c);
        const int pos = nc + __popc(bj & lt);
        if (c && pos < cap) cand[pos] = key[j];
        nc += __popc(bj);
    }
    nc = min(nc, cap);
    __syncwarp();
    for (int ci = lane; ci < nc; ci += 32) {
        const unsigned long long mine = cand[ci];
        int rank = 0;
#pragma unroll 4
        for (int q = 0; q < nc; ++q) rank += cand[q] > mine;
        if (rank < k) {
            sel_e[rank] = route_key_expert(mine);
            sel_w[rank] = route_key_value(mine);
        }
    }
    __syncwarp();
    return __any_sync(FULL, nan);
}

FE_DEV bool warp_route(const float* row, int E, int k, int lane, unsigned long long* cand, int cap, int* sel_e,
                       float* sel_w)
{
    if (E <= 32) return warp_topk<1>(row, E, k, lane, cand, cap, sel_e, sel_w);
    if (E <= 64) return warp_topk<2>(row, E, k, lane, cand, cap, sel_e, sel_w);
    if (E <= 128) return warp_topk<4>(row, E, k, lane, cand, cap, sel_e, sel_w);
    if (E <= 256) return warp_topk<8>(row, E, k, lane, cand, cap, sel_e, sel_w);
    return warp_topk<16>(row, E, k, lane, cand, cap, sel_e, sel_w);
}

// Softmax of one token's k selected logits (slot order) in place, by one warp.
FE_DEV void warp_softmax(float* sel_w, int k, int lane)
{
    const float l0 = sel_w[0];
    const float ej = lane < k ? expf(sel_w[lane] - l0) : 0.0f;
    const float ssum = warp_sum(ej);
    __syncwarp();
    if (lane < k) sel_w[lane] = ej / ssum;
    __syncwarp();
}

}  // namespace fe
