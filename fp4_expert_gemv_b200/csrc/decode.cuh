// Fused small-T decode layer: one launch per layer.
//
// "FireEcho Engine", sections "Speed Optimization History" (single-token
// decode fast path, multi-expert kernel, packed contiguous expert buffer,
// CUDA-graph decode) and "The Goliath Kernel: Why It's Fast" (expert IDs read
// on the GPU, FP4 dequantised in registers, tensor-core accumulation, nothing
// dequantised written to memory).  The pages' kernel runs one Triton launch
// per projection; here the whole layer is one launch, so that the HBM stream
// of the down weights overlaps the gate_up work and no launch boundary sits
// inside the layer:
//
//   1. every CTA routes the T tokens itself (one warp per token: warp top-k
//      over orderable keys, ties to the lower index, softmax over the k
//      selected) and groups the T*k pairs by expert; CTA 0 publishes the
//      routing; a bulk copy brings the x rows into shared memory meanwhile;
//   2. from the number of distinct routed experts every CTA reads, in a
//      table built at reserve time, its range of gate_up units (16 gate + 16
//      up columns of one routed expert) and its range of down units (16
//      output columns over all routed experts), balanced in bytes;
//   3. one warp issues cp.async.bulk copies of the CTA's gate_up units into
//      shared memory, one mbarrier per unit; the down units follow once the
//      first gate_up unit has landed, so the bytes the exchange waits for
//      come first;
//   4. gate_up units: mma.m16n8k16 with the tokens of the unit's expert as
//      the N columns (mma.cuh); the per-warp partials of all units wait in
//      shared memory for one reduction, which writes SiLU(gate)*up to global
//      memory (L2) as 64-bit words holding the fp32 value and the launch's tag;
//      then the CTA adds 1 to an arrival counter;
//   5. each CTA that owns down units polls the counter (one thread) until all
//      but a few CTAs have arrived, then reads act back; a word carrying this
//      launch's tag is this launch's value (the data is its own ready flag),
//      and only words without it are read again;
//   6. down units: the routed experts' quads spread over all warps, the
//      pairs as the N columns; the 16 outputs of every pair are combined in
//      slot order, so y is written once, without atomics.
//
// The kernel is launched with programmatic dependent launch: its CTAs load
// only static data before griddepcontrol.wait, so the next layer's CTAs can
// be resident and waiting while this layer finishes.
#pragma once

#include <vector>

#include "common.cuh"
#include "mma.cuh"

namespace fe {

constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kDecMaxPairs = 16;   // T * top_k handled by the fused kernel
constexpr int kDecMaxItems = 48;   // weight units (mbarriers) per CTA
constexpr int kDecMaxE = 512;      // experts routed by one warp: 16 logits per lane
constexpr int kDecQuadsPerWarp = 4;   // gate_up quads whose x fragments a warp keeps in registers
constexpr int kDecCandCap = 128;   // candidate keys per routing warp (in the gate_up partials' space)
constexpr int kDecRedFloats = 4096;   // gate_up partials held before one reduction (also the down partials)
constexpr int kDecArriveSlack = 16;   // producers still out when consumers start reading act
constexpr int kDecMaxJobs = kDecRedFloats / (kDecWarps * 32);   // act columns one reduction serves
constexpr int kDecDownLate = 1;   // down copies issued once this many gate_up units landed (0: at once)
constexpr uint32_t kDevBarrierTimeout = 0x4;
constexpr uint32_t kDevLoadTimeout = 0x8;

struct DecodeParams {
    const uint16_t* x;        // bf16 [T][H]
    const float* logits;      // [T][E]
    uint16_t* y;              // bf16 [T][H]
    int T, E, H, I, k;
    const uint8_t* gu_blocks; // [E][I/16] gate_up units of 2 blocks (18H bytes)
    const uint8_t* dn_blocks; // [E][H/16] down blocks (9I bytes)
    const int32_t* plan;      // [kDecMaxPairs + 1][2][grid + 1]: first gate_up / down unit of each CTA, per nd
    int32_t* idx;
    float* w;
    int32_t* counts;
    int32_t* offsets;
    int32_t* sorted_pair;
    int32_t* pair_row;
    unsigned long long* act;  // [kDecMaxPairs][I] by pair id: (launch tag << 32) | fp32 bits
    unsigned long long* epoch;  // [grid + 1]: launches CTA c has run on this handle; [grid]: arrivals
    uint32_t* status;
    unsigned long long timeout_ns;  // bound of every wait
    uint32_t weight_bytes;    // shared memory reserved for weight units
    int bulk_inputs;          // x and logits rows copied with cp.async.bulk (16-byte aligned)
    unsigned long long* trace;  // optional [grid][64]: %globaltimer (0-31) and clock64 (32-63) stamps of the phases
};

// ---- work split (host only: the kernel reads the table) ---------------------------
// gate_up units: nd * I/16 of 18H bytes; down units: H/16 of nd * 9I bytes.
// gate_up units are spread evenly over the CTAs; then each down unit goes to
// the CTA with the fewest bytes so far (lowest index on ties).  Returns, for
// c = 0..grid, the first gate_up and the first down unit of CTA c.
inline void decode_split(int nd, int H, int I, int grid, std::vector<int>& gu_first, std::vector<int>& dn_first)
{
    const int n_gu = nd * (I / 16), n_dn = H / 16;
    const int64_t gu_bytes = 18ll * H, dn_bytes = (int64_t)nd * 9 * I;
    std::vector<int> cgu(grid), cdn(grid, 0);
    std::vector<int64_t> load(grid);
    for (int c = 0; c < grid; ++c) {
        cgu[c] = (int)((int64_t)(c + 1) * n_gu / grid - (int64_t)c * n_gu / grid);
        load[c] = cgu[c] * gu_bytes;
    }
    for (int j = 0; j < n_dn; ++j) {
        int best = 0;
        for (int c = 1; c < grid; ++c)
            if (load[c] < load[best]) best = c;
        cdn[best] += 1;
        load[best] += dn_bytes;
    }
    gu_first.assign(grid + 1, 0);
    dn_first.assign(grid + 1, 0);
    for (int c = 0; c < grid; ++c) {
        gu_first[c + 1] = gu_first[c] + cgu[c];
        dn_first[c + 1] = dn_first[c] + cdn[c];
    }
}

// ---- PTX wrappers --------------------------------------------------------------
FE_DEV uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

FE_DEV void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

FE_DEV void mbar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

FE_DEV bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for phase 0 of a one-shot barrier, at most timeout_ns; false on timeout.
FE_DEV bool mbar_wait0(uint32_t bar, unsigned long long timeout_ns)
{
    if (mbar_try_wait(bar, 0)) return true;
    const unsigned long long t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait(bar, 0)) return true;
        if (globaltimer_ns() - t0 > timeout_ns) return false;
    }
}

FE_DEV void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

// Phase stamp i of the optional trace: %globaltimer and the SM's cycle counter.
FE_DEV void stamp(unsigned long long* trace, int i)
{
    asm volatile("" ::: "memory");
    trace[i] = globaltimer_ns();
    trace[32 + i] = (unsigned long long)clock64();
    asm volatile("" ::: "memory");
}

// The act exchange.  act words carry the launch's tag next to the value
// (each 64-bit word is single-copy atomic, so a reader sees the old tag or the
// new value): a word with this launch's tag is this launch's value, whatever
// order the memory system delivers things in.  So that consumers do not flood
// L2 with polls of data that is not there yet, every CTA also adds 1 to an
// arrival counter after its act stores, and a consumer reads act only once the
// counter shows every CTA of the launch; the counter carries no ordering (no
// fence), the tags still decide, and the few words still in flight are read again.
FE_DEV void st_relaxed_u64(unsigned long long* p, unsigned long long v)
{
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

FE_DEV void ld_relaxed_2u64(const unsigned long long* p, unsigned long long& a, unsigned long long& b)
{
    asm volatile("ld.relaxed.gpu.global.v2.u64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "l"(p) : "memory");
}

FE_DEV void arrive_relaxed(unsigned long long* counter)
{
    asm volatile("red.relaxed.gpu.global.add.u64 [%0], 1;" ::"l"(counter) : "memory");
}

FE_DEV unsigned long long ld_relaxed_u64(const unsigned long long* p)
{
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// Act tag of launch ep (1, 2, ...): never 0 (the value act starts from) and
// different for consecutive launches, also across the wrap of 32 bits.
FE_DEV unsigned act_tag(unsigned long long ep) { return (unsigned)(ep % 0xffffffffull) + 1u; }

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

struct DecodeShared {
    int sel_e[kDecMaxPairs];
    float sel_w[kDecMaxPairs];
    int sp[kDecMaxPairs];         // pair ids in (expert, pair) order
    int pdi[kDecMaxPairs];        // pair -> distinct-expert index
    int dex[kDecMaxPairs];        // distinct experts, ascending
    int dstart[kDecMaxPairs + 1]; // first sorted position of each distinct expert
    int plan[kDecMaxPairs + 1][4];  // per nd: gate_up first/end, down first/end of this CTA
    int xshift[kDecMaxPairs];
    int job_act[kDecMaxJobs];     // pending act columns: act offset (pair row, unit block),
    int job_red[kDecMaxJobs];     // first partial, partial stride between warps, x shift
    int job_stride[kDecMaxJobs];
    int job_shift[kDecMaxJobs];
    int ashift[kDecMaxPairs];
    int item_d[kDecMaxPairs + 1];   // down items: (distinct expert, first sorted pair, pairs <= 8)
    int item_r[kDecMaxPairs + 1];
    int item_n[kDecMaxPairs + 1];
    int n_items;
    int nd;
    int abort;
    unsigned long long target;    // arrivals that complete this launch's act
    unsigned tag;                 // this launch's act tag
    float wmax[2][kDecWarps];
    float ob[kDecMaxPairs * 16];  // down: [pair][16] outputs
};


// Single-token grouping: k distinct experts, the sorted position of slot
// `lane` is the number of selected experts below its own.
FE_DEV void group_single_token(DecodeShared& S, int k, int lane)
{
    if (lane < k) {
        const int ep = S.sel_e[lane];
        int pos = 0;
#pragma unroll 4
        for (int q = 0; q < k; ++q) pos += S.sel_e[q] < ep;
        S.sp[pos] = lane;
        S.pdi[lane] = pos;
        S.dex[pos] = ep;
        S.dstart[pos] = pos;
        S.item_d[pos] = pos;
        S.item_r[pos] = pos;
        S.item_n[pos] = 1;
    }
    if (lane == 0) {
        S.nd = k;
        S.dstart[k] = k;
        S.n_items = k;
    }
    __syncwarp();
}

// Bulk copies of the CTA's down units (one per routed expert and unit), issued
// by the lanes of one warp; their barriers' byte counts are already armed.
FE_DEV void issue_down(const DecodeParams& p, const DecodeShared& S, uint32_t dst, int nd, int dn0, int ndn, int ngu,
                       uint32_t dn_blk, uint32_t mbar0, int lane)
{
    for (int i = lane; i < ndn * nd; i += 32) {
        const int u = i / nd, dd = i - u * nd, j = dn0 + u;
        bulk_g2s(dst + (u * nd + dd) * dn_blk, p.dn_blocks + ((size_t)S.dex[dd] * (p.H / 16) + j) * dn_blk, dn_blk,
                 mbar0 + 8 * (ngu + u));
    }
}

// Byte offsets of the dynamic shared memory regions.
struct DecodeSmem {
    uint32_t mbar, shared, red, dred, xs, as, xr, total;
};

__host__ __device__ inline uint32_t align16(uint32_t v) { return (v + 15u) & ~15u; }

// xs: T x rows + 1 zero row; as: T*k act rows + 1 zero row (brow_words each).
__host__ __device__ inline DecodeSmem decode_smem_layout(uint32_t weight_bytes, int T, int k, int H, int I, int E)
{
    DecodeSmem L;
    L.mbar = weight_bytes;
    L.shared = L.mbar + 8 * (kDecMaxItems + 1);
    L.red = align16(L.shared + (uint32_t)sizeof(DecodeShared));
    L.dred = L.red;   // gate_up partials and down partials are never live together
    static_assert(kDecRedFloats >= kDecWarps * 32 * 8 && kDecRedFloats >= 8 * 4 * 32 * 4, "partials space");
    static_assert(kDecRedFloats * 4 >= kDecWarps * kDecCandCap * 8, "routing candidates space");
    L.xs = L.red + 4u * kDecRedFloats;
    L.as = L.xs + 4u * (T + 1) * brow_words(H);
    L.xr = align16(L.as + 4u * (T * k + 1) * brow_words(I));
    L.total = align16(L.xr + 2u * T * H);
    return L;
}

__global__ void __launch_bounds__(kDecThreads, 1) decode_kernel(DecodeParams p)
{
    extern __shared__ __align__(128) uint8_t dsm[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2;
    const int T = p.T, E = p.E, H = p.H, I = p.I, k = p.k, P = T * k;
    const DecodeSmem L = decode_smem_layout(p.weight_bytes, T, k, H, I, E);
    const uint32_t gu_unit = 2u * block_bytes(H), dn_blk = block_bytes(I);
    const int xrw = brow_words(H), arw = brow_words(I);

    uint8_t* wbuf = dsm;
    DecodeShared& S = *reinterpret_cast<DecodeShared*>(dsm + L.shared);
    float* red = reinterpret_cast<float*>(dsm + L.red);
    float* dred = reinterpret_cast<float*>(dsm + L.dred);   // down partials [8 items][4 quarters][lane][4]
    uint32_t* xs = reinterpret_cast<uint32_t*>(dsm + L.xs);
    uint32_t* as = reinterpret_cast<uint32_t*>(dsm + L.as);
    uint16_t* xr = reinterpret_cast<uint16_t*>(dsm + L.xr);
    const uint32_t mbar0 = smem_addr(dsm + L.mbar);
    const uint32_t in_bar = mbar0 + 8 * kDecMaxItems;
    const bool tracing = p.trace != nullptr;
    unsigned long long* trace = tracing ? p.trace + (size_t)blockIdx.x * 64 : nullptr;
    if (tracing && tid == 0) stamp(trace, 0);

    // ---- 0. static data only, then wait for the previous grid ---------------------
    if (tid >= 64 && tid < 64 + 4 * (kDecMaxPairs + 1)) {
        // (warps 2-4: the routing warp goes straight to the logits)
        const int nd = (tid - 64) >> 2, which = tid & 3;   // 0: gate_up first, 1: end, 2: down first, 3: end
        const int32_t* row = p.plan + ((size_t)nd * 2 + (which >> 1)) * (gridDim.x + 1);
        S.plan[nd][which] = row[blockIdx.x + (which & 1)];
    }
    if (warp == 1) {
        // lane 16 initialises in_bar (index kDecMaxItems) and issues the x copy below
        for (int u = lane; u <= kDecMaxItems; u += 32) mbar_init(mbar0 + 8 * u, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        if (lane == 0) S.abort = 0;
    }
    for (int i = tid; i < xrw; i += kDecThreads) xs[T * xrw + i] = 0u;       // zero B rows
    for (int i = tid; i < arw; i += kDecThreads) as[P * arw + i] = 0u;
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (tracing && tid == 0) stamp(trace, 8);
    if (warp == 1 && lane == 16 && p.bulk_inputs) {
        const uint32_t xb = 2u * T * H;
        mbar_expect_tx(in_bar, xb);
        bulk_g2s(smem_addr(xr), p.x, xb, in_bar);
    }
    // this launch's arrival target: every launch runs every CTA (the grid is
    // fixed per handle) and each CTA arrives once, so the per-CTA launch counts
    // move in lockstep and all CTAs derive the same target without talking to
    // each other; the load is consumed only when the staging warps finish
    unsigned long long ep_e0 = 0;
    if (tid == kDecThreads - 1) ep_e0 = *reinterpret_cast<volatile unsigned long long*>(p.epoch + blockIdx.x);
    // candidate keys of the routing warps live in the gate_up partials' space
    const int nroute = min(T, kDecWarps);
    const int cap = (kDecWarps * kDecCandCap) / nroute;
    unsigned long long* cand = reinterpret_cast<unsigned long long*>(red) + warp * cap;

    // ---- 1. routing: warp t selects the top-k logits of token t ----------------------
    // With T = 1, warp 0 routes and hands the selection to warp 1, which groups
    // and issues the loads (a warp fresh from the divergent selection code ran
    // the short serial steps after it several times slower); the softmax and the
    // published routing come after.  With T > 1 every token's warp also takes its
    // softmax, then the CTA meets before the grouping.
    if (warp < nroute) {
        for (int t = warp; t < T; t += kDecWarps) {
            const bool nan = warp_route(p.logits + (size_t)t * E, E, k, lane, cand, cap, S.sel_e + t * k, S.sel_w + t * k);
            if (nan && lane == 0 && blockIdx.x == 0) atomicOr(p.status, kDevNanLogit);
            if (T > 1) warp_softmax(S.sel_w + t * k, k, lane);
        }
        if (T == 1) asm volatile("bar.arrive 3, 64;" ::: "memory");
    }
    if (tracing && tid == 0) stamp(trace, 10);
    if (T > 1) __syncthreads();
    if (tracing && tid == 0) stamp(trace, 12);

    if (warp == 1) {
        // ---- 2. grouping: stable order of the P pairs by expert --------------------------
        if (T == 1) {
            asm volatile("bar.sync 3, 64;" ::: "memory");
            group_single_token(S, k, lane);
        } else {
            const int ep = lane < P ? S.sel_e[lane] : 0x7fffffff;
            uint32_t less = 0, same = 0;
            for (int q = 0; q < P; ++q) {
                const int eq = __shfl_sync(0xffffffffu, ep, q);
                less |= (uint32_t)(eq < ep) << q;
                same |= (uint32_t)(eq == ep) << q;
            }
            const uint32_t below = (1u << lane) - 1u;
            const int rank = __popc(less) + __popc(same & below);   // sorted position of pair `lane`
            const bool first = lane < P && (same & below) == 0;     // lowest pair id of its expert
            const uint32_t firsts = __ballot_sync(0xffffffffu, first);
            const int dless = __popc(firsts & less);                // distinct index of its expert
            const int nd = __popc(firsts);
            const int cnt = __popc(same);                           // pairs of its expert
            const int nit = first ? (cnt + 7) / 8 : 0;              // down items (<= 8 pairs each)
            int ibase = 0, n_items = 0;
            for (int q = 0; q < P; ++q) {
                const int nq = __shfl_sync(0xffffffffu, nit, q);
                ibase += ((less >> q) & 1u) ? nq : 0;
                n_items += nq;
            }
            if (lane < P) {
                S.sp[rank] = lane;
                S.pdi[lane] = dless;
            }
            if (first) {
                S.dex[dless] = ep;
                S.dstart[dless] = rank;
                for (int i = 0; i < nit; ++i) {
                    S.item_d[ibase + i] = dless;
                    S.item_r[ibase + i] = rank + 8 * i;
                    S.item_n[ibase + i] = min(8, cnt - 8 * i);
                }
            }
            if (lane == 0) {
                S.nd = nd;
                S.dstart[nd] = P;
                S.n_items = n_items;
            }
        }
        __syncwarp();
        if (tracing && lane == 0) stamp(trace, 9);
        // the staging warps were parked until now, so that the path to the loads had
        // the SM to itself; the copy issue below is paced by the TMA unit
        asm volatile("bar.arrive 2, %0;" ::"n"(kDecThreads - 32) : "memory");

        // ---- 3. every weight load of this CTA, issued now ------------------------------
        {
            const int nd = S.nd;
            const int ntu = I / 16;   // gate_up units per expert
            const int gu0 = S.plan[nd][0], ngu = S.plan[nd][1] - gu0;
            const int dn0 = S.plan[nd][2], ndn = S.plan[nd][3] - dn0;
            const uint32_t dn_unit = (uint32_t)nd * dn_blk;
            for (int u = lane; u < ngu + ndn; u += 32) mbar_expect_tx(mbar0 + 8 * u, u < ngu ? gu_unit : dn_unit);
            __syncwarp();
            if (tracing && lane == 0) stamp(trace, 15);
            const uint32_t wb = smem_addr(wbuf);
            for (int u = lane; u < ngu; u += 32) {
                const int gid = gu0 + u, dd = gid / ntu, j = gid - dd * ntu;
                bulk_g2s(wb + u * gu_unit, p.gu_blocks + ((size_t)S.dex[dd] * ntu + j) * gu_unit, gu_unit,
                         mbar0 + 8 * u);
            }
            if (kDecDownLate == 0 || ngu == 0) issue_down(p, S, wb + ngu * gu_unit, nd, dn0, ndn, ngu, dn_blk, mbar0, lane);
        }
        if (tracing && lane == 0) stamp(trace, 1);
    } else if (warp == 0) {
        // ---- the routing's remaining outputs ------------------------------------------------
        if (T == 1) warp_softmax(S.sel_w, k, lane);
        if (blockIdx.x == 0) {
            for (int q = lane; q < P; q += 32) {
                p.idx[q] = S.sel_e[q];
                p.w[q] = S.sel_w[q];
            }
        }
    } else {
        asm volatile("bar.sync 2, %0;" ::"n"(kDecThreads - 32) : "memory");
        // ---- 4. (warps 2..) x rows as fp16 pairs with a power-of-two shift per token -----
        constexpr int XT = kDecThreads - 64;
        const int xt = tid - 64;
        if (blockIdx.x == 0) {
            for (int e = xt; e <= E; e += XT) {
                int below = 0, eq = 0;
                for (int q = 0; q < P; ++q) {
                    below += S.sel_e[q] < e;
                    eq += S.sel_e[q] == e;
                }
                p.offsets[e] = below;
                if (e < E) p.counts[e] = eq;
            }
            for (int r = xt; r < P; r += XT) {
                p.sorted_pair[r] = S.sp[r];
                p.pair_row[S.sp[r]] = r;
            }
        }
        // every thread of the group waits (bounded) for x; the group agrees on the
        // outcome before the named barriers of the staging loop
        if (p.bulk_inputs && !mbar_wait0(in_bar, p.timeout_ns)) S.abort = 1;
        asm volatile("bar.sync 1, %0;" ::"n"(XT) : "memory");
        if (S.abort) {
            if (xt == 0) atomicOr(p.status, kDevLoadTimeout);
        } else {
            for (int t = 0; t < T; ++t) {
                const uint32_t* xw = p.bulk_inputs ? reinterpret_cast<const uint32_t*>(xr + (size_t)t * H)
                                                   : reinterpret_cast<const uint32_t*>(p.x + (size_t)t * H);
                float m = 0.0f;
                for (int r = xt; r < H / 2; r += XT) {
                    const uint32_t two = xw[r];
                    m = fmaxf(m, fmaxf(fabsf(bf16_bits_to_f32((uint16_t)(two & 0xffff))),
                                       fabsf(bf16_bits_to_f32((uint16_t)(two >> 16)))));
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                if (lane == 0) S.wmax[t & 1][warp] = m;
                asm volatile("bar.sync 1, %0;" ::"n"(XT) : "memory");
                float mm = 0.0f;
#pragma unroll
                for (int w2 = 2; w2 < kDecWarps; ++w2) mm = fmaxf(mm, S.wmax[t & 1][w2]);
                const int sh = fp16_shift(mm);
                const float scl = pow2f(-sh);
                if (xt == 0) S.xshift[t] = sh;
                for (int r = xt; r < H / 2; r += XT) {
                    const uint32_t two = xw[r];
                    xs[t * xrw + bfrag_word(r)] = f32x2_to_f16x2_rn(bf16_bits_to_f32((uint16_t)(two & 0xffff)) * scl,
                                                                   bf16_bits_to_f32((uint16_t)(two >> 16)) * scl);
                }
            }
        }
        if (tracing && xt == 0) stamp(trace, 2);
        if (tid == kDecThreads - 1) {
            S.target = (ep_e0 + 1ull) * gridDim.x;
            S.tag = act_tag(ep_e0 + 1ull);
            p.epoch[blockIdx.x] = ep_e0 + 1ull;
        }
    }
    __syncthreads();
    const int nd = S.nd;
    const int ntu = I / 16;   // gate_up units per expert
    const int gu0 = S.plan[nd][0], gu1 = S.plan[nd][1], dn0 = S.plan[nd][2], dn1 = S.plan[nd][3];
    const int ngu = gu1 - gu0, ndn = dn1 - dn0;
    const uint32_t dn_unit = (uint32_t)nd * dn_blk;
    if (tracing && tid == 0) {
        trace[32 + 28] = (unsigned long long)ngu;
        trace[32 + 29] = (unsigned long long)ndn;
    }

    // ---- 5. gate_up units -> act -------------------------------------------------------
    // Warp w runs quads w, w + W, ... (W = warps) of every unit.  Its x fragments
    // for those quads stay in registers while the n-block's rows stay the same
    // (always, for one token): the inner loop then reads only weights.  The
    // per-warp partials of a tile (one unit, up to 8 tokens) wait in shared
    // memory, and one reduction serves every tile computed since the last, so
    // the warps meet once per layer rather than once per unit; act is read
    // only after every CTA has written its part, so nothing waits on it sooner.
    uint32_t off = 0;
    {
        const int nq = H / 64;
        constexpr int QPW = kDecQuadsPerWarp;
        const int npass = (nq + QPW * kDecWarps - 1) / (QPW * kDecWarps);
        uint32_t bx[QPW][8];
        int bkey = -1;
        int njobs = 0, red_used = 0;   // the same in every thread
        const unsigned long long tg = (unsigned long long)S.tag << 32;
        // reduce the pending act columns' partials over the warps and write act
        auto flush = [&]() {
            __syncthreads();
            if (tracing && tid == 0) stamp(trace, 17);
            if (!*reinterpret_cast<volatile int*>(&S.abort)) {
                const int half = lane & 1, n = lane >> 1;
                for (int jb = warp; jb < njobs; jb += kDecWarps) {
                    const float* rw = red + S.job_red[jb] + half * (kDecWarps / 2) * S.job_stride[jb] + n;
                    const int stride = S.job_stride[jb];
                    float gs = 0.0f, us = 0.0f;
#pragma unroll
                    for (int w2 = 0; w2 < kDecWarps / 2; ++w2) {
                        gs += rw[w2 * stride];
                        us += rw[w2 * stride + 16];
                    }
                    gs += __shfl_xor_sync(0xffffffffu, gs, 1);
                    us += __shfl_xor_sync(0xffffffffu, us, 1);
                    if (half == 0) {
                        const float m = pow2f(S.job_shift[jb]);
                        const float a = silu_mul_fast(gs * m, us * m);
                        st_relaxed_u64(p.act + S.job_act[jb] + n, tg | __float_as_uint(a));
                    }
                }
            }
            if (tracing && tid == 0) stamp(trace, 18);
            __syncthreads();
            if (tracing && tid == 0) stamp(trace, 19);
            njobs = 0;
            red_used = 0;
        };
        for (int u = 0; u < ngu; ++u) {
            // after a timed-out wait the other units are skipped (their work is
            // discarded at the reduction, which every thread still reaches)
            if (*reinterpret_cast<volatile int*>(&S.abort) || !mbar_wait0(mbar0 + 8 * u, p.timeout_ns)) {
                if (!S.abort) atomicOr(p.status, kDevLoadTimeout);
                S.abort = 1;
            }
            if (tracing && tid == 0 && (u == 0 || u == ngu - 1)) stamp(trace, u == 0 ? 11 : 13);
            if (tracing && tid == 0 && u == 1) stamp(trace, 24);
            if (kDecDownLate > 0 && warp == 1 && u == min(ngu, kDecDownLate) - 1)
                issue_down(p, S, smem_addr(wbuf) + ngu * gu_unit, nd, dn0, ndn, ngu, dn_blk, mbar0, lane);
            const int gid = gu0 + u, dd = gid / ntu, j = gid - dd * ntu;
            const uint8_t* blk0 = wbuf + off;
            const uint8_t* blk1 = blk0 + block_bytes(H);
            const int r0 = S.dstart[dd], r1 = S.dstart[dd + 1];
            for (int nb = r0; nb < r1; nb += 8) {
                const int nvalid = min(8, r1 - nb);
                const int need = kDecWarps * nvalid * 32;
                if (red_used + need > kDecRedFloats) flush();
                const int key = T == 1 ? 0 : (dd << 8) + (nb - r0);
                const uint32_t* brow = xs + (g < nvalid ? S.sp[nb + g] / k : T) * xrw;
                float t0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, t1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                if (nq == QPW * kDecWarps) {
                    // one pass, every quad of the warp valid: fixed offsets, no selects
                    if (key != bkey) {
#pragma unroll
                        for (int i = 0; i < QPW; ++i) load_bfrag(brow, warp + kDecWarps * i, lane, bx[i]);
                        bkey = key;
                    }
#pragma unroll
                    for (int i = 0; i < QPW; ++i) quad_mma2_b(blk0, blk1, H, bx[i], warp + kDecWarps * i, lane, t0, t1);
                } else
                for (int pass = 0; pass < npass; ++pass) {
                    const int qbase = pass * QPW * kDecWarps + warp;
                    // quads past nq (H not a multiple of 64 QPW W) repeat quad qbase with a
                    // zero B, so the unrolled body has no branches between its quads
                    if (key != bkey || npass > 1) {
#pragma unroll
                        for (int i = 0; i < QPW; ++i) {
                            const bool ok = qbase + kDecWarps * i < nq;
                            load_bfrag(ok ? brow : xs + T * xrw, ok ? qbase + kDecWarps * i : 0, lane, bx[i]);
                        }
                        bkey = key;
                    }
                    if (qbase < nq) {
#pragma unroll
                        for (int i = 0; i < QPW; ++i) {
                            const int q = qbase + kDecWarps * i < nq ? qbase + kDecWarps * i : qbase;
                            quad_mma2_b(blk0, blk1, H, bx[i], q, lane, t0, t1);
                        }
                    }
                }
                if (tracing && tid == 0 && u < 2) stamp(trace, u == 0 ? 16 : 25);
                // partials of the valid token columns only: [warp][column][gate 16 | up 16];
                // lane (g, c) holds rows g, g+8 of columns 2c, 2c+1
                {
                    const int c = lane & 3;
                    float* rw = red + red_used + warp * nvalid * 32;
                    if (2 * c < nvalid) {
                        rw[(2 * c) * 32 + g] = t0[0];
                        rw[(2 * c) * 32 + g + 8] = t0[2];
                        rw[(2 * c) * 32 + 16 + g] = t1[0];
                        rw[(2 * c) * 32 + 24 + g] = t1[2];
                    }
                    if (2 * c + 1 < nvalid) {
                        rw[(2 * c + 1) * 32 + g] = t0[1];
                        rw[(2 * c + 1) * 32 + g + 8] = t0[3];
                        rw[(2 * c + 1) * 32 + 16 + g] = t1[1];
                        rw[(2 * c + 1) * 32 + 24 + g] = t1[3];
                    }
                }
                if (tid < nvalid) {
                    // column tid of this tile: its act word, partials and x shift
                    const int pid = S.sp[nb + tid];
                    S.job_act[njobs + tid] = pid * I + 16 * j;
                    S.job_red[njobs + tid] = red_used + tid * 32;
                    S.job_stride[njobs + tid] = nvalid * 32;
                    S.job_shift[njobs + tid] = S.xshift[pid / k];
                }
                njobs += nvalid;
                red_used += need;
            }
            off += gu_unit;
        }
        flush();
    }
    // every CTA arrives once per launch, on every path, so the counts stay in lockstep
    if (tid == 0) arrive_relaxed(p.epoch + gridDim.x);
    if (tracing && tid == 0) stamp(trace, 3);
    if (tracing) {
        // diagnostics only: when the down weights have landed
        for (int u = 0; u < ndn; ++u) mbar_wait0(mbar0 + 8 * (ngu + u), p.timeout_ns);
        if (tid == 0) stamp(trace, 14);
    }

    // ---- 6. down units: read every CTA's act back (tagged), compute, combine -----------
    off = (uint32_t)ngu * gu_unit;
    if (ndn > 0 && !S.abort) {
        const unsigned long long t_poll = globaltimer_ns();
        if (tid == 0) {
            // one thread polls the arrival counter (bounded) until all but the last
            // few CTAs have arrived; the CTA meets after it and reads act, polling
            // only the words those few CTAs still have to deliver
            const unsigned long long target = S.target;
            const unsigned long long* ctr = p.epoch + gridDim.x;
            while ((long long)(ld_relaxed_u64(ctr) - (target - kDecArriveSlack)) < 0) {
                if (globaltimer_ns() - t_poll > p.timeout_ns) {
                    atomicOr(p.status, kDevBarrierTimeout);
                    S.abort = 1;
                    break;
                }
            }
            if (tracing) stamp(trace, 26);
        }
        __syncthreads();
        const unsigned tag = S.tag;
        // warp pp stages pair pp: up to 16 chunks of two tagged words per lane, all
        // requested at once, then only the ones not yet carrying this launch's tag
        // again; the values are kept, the tags only checked
        for (int pp = warp; pp < P && !S.abort; pp += kDecWarps) {
            const unsigned long long* src = p.act + (size_t)pp * I;
            float v0[16], v1[16];
            uint32_t pending = 0;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int r = lane + 32 * i;
                unsigned long long w0 = 0ull, w1 = 0ull;
                if (2 * r < I) {
                    ld_relaxed_2u64(src + 2 * r, w0, w1);
                    if ((unsigned)(w0 >> 32) != tag || (unsigned)(w1 >> 32) != tag) pending |= 1u << i;
                }
                v0[i] = __uint_as_float((uint32_t)w0);
                v1[i] = __uint_as_float((uint32_t)w1);
            }
            bool late = false;
            if (tracing && lane == 0 && pp == 0) stamp(trace, 22);
            int rounds = 0;
            while (__any_sync(0xffffffffu, pending != 0) && !late) {
                ++rounds;
                __nanosleep(32);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    if ((pending >> i) & 1u) {
                        unsigned long long w0, w1;
                        ld_relaxed_2u64(src + 2 * (lane + 32 * i), w0, w1);
                        if ((unsigned)(w0 >> 32) == tag && (unsigned)(w1 >> 32) == tag) pending &= ~(1u << i);
                        v0[i] = __uint_as_float((uint32_t)w0);
                        v1[i] = __uint_as_float((uint32_t)w1);
                    }
                }
                late = __any_sync(0xffffffffu, globaltimer_ns() - t_poll > p.timeout_ns);
            }
            if (late && lane == 0) {
                atomicOr(p.status, kDevBarrierTimeout);
                S.abort = 1;
            }
            if (tracing && lane == 0 && pp == 0) {
                stamp(trace, 23);
                trace[27] = rounds;
            }
            float m = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) m = fmaxf(m, fmaxf(fabsf(v0[i]), fabsf(v1[i])));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            const int sh = fp16_shift(m);
            const float scl = pow2f(-sh);
            if (lane == 0) S.ashift[pp] = sh;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int r = lane + 32 * i;
                if (2 * r < I) as[pp * arw + bfrag_word(r)] = f32x2_to_f16x2_rn(v0[i] * scl, v1[i] * scl);
            }
        }
        __syncthreads();
    }
    if (tracing && tid == 0) stamp(trace, 4);
    for (int u = 0; u < ndn; ++u) {
        const uint32_t bar = mbar0 + 8 * (ngu + u);
        if (!mbar_wait0(bar, p.timeout_ns)) {
            if (tid == 0) { atomicOr(p.status, kDevLoadTimeout); S.abort = 1; }
        }
        __syncthreads();
        if (tracing && tid == 0 && u == 0) stamp(trace, 6);
        const int j = dn0 + u;
        if (!S.abort) {
            // every warp runs a strided share of the 64-k quads for every routed
            // expert (independent accumulator chains); partial sums go to dred,
            // then warp dd adds the 8 warps' partials of expert dd in warp order
            const int nq = I / 64;
            const int n_items = S.n_items;
            for (int i0 = 0; i0 < n_items; i0 += 8) {
                const int dn = min(8, n_items - i0);
                // 32 tasks = 8 items x 4 quarters of K; warp w runs tasks w + W*m:
                // items (w/4) + (W/4)*m, all in quarter w % 4 (independent chains)
                constexpr int TPW = 32 / kDecWarps;   // tasks per warp
                const int quarter = warp & 3;
                const int qa = quarter * nq / 4, qb = (quarter + 1) * nq / 4;
                float tot[TPW][4];
#pragma unroll
                for (int m = 0; m < TPW; ++m)
#pragma unroll
                    for (int c2 = 0; c2 < 4; ++c2) tot[m][c2] = 0.0f;
                // the tasks' B rows and weight blocks, resolved once; tasks past the last
                // item redo item i0 and are not stored, so the body has no branches
                const uint32_t* brow[TPW];
                const uint8_t* dblk[TPW];
#pragma unroll
                for (int m = 0; m < TPW; ++m) {
                    const int i = (warp >> 2) + (kDecWarps / 4) * m;
                    const int it = i0 + (i < dn ? i : 0);
                    const int r0 = S.item_r[it], nvalid = S.item_n[it];
                    brow[m] = as + (g < nvalid ? S.sp[r0 + g] : P) * arw;
                    dblk[m] = wbuf + off + S.item_d[it] * dn_blk;
                }
                for (int q = qa; q < qb; ++q) {
                    uint32_t b[TPW][8];
#pragma unroll
                    for (int m = 0; m < TPW; ++m) load_bfrag(brow[m], q, lane, b[m]);
#pragma unroll
                    for (int m = 0; m < TPW; ++m) quad_mma_b(dblk[m], I, b[m], q, lane, tot[m]);
                }
#pragma unroll
                for (int m = 0; m < TPW; ++m) {
                    const int i = (warp >> 2) + (kDecWarps / 4) * m;
                    if (i < dn)
#pragma unroll
                        for (int c2 = 0; c2 < 4; ++c2) dred[((i * 4 + quarter) * 32 + lane) * 4 + c2] = tot[m][c2];
                }
                if (tracing && tid == 0 && u == 0 && i0 == 0) stamp(trace, 20);
                __syncthreads();
                if (tracing && tid == 0 && u == 0 && i0 == 0) stamp(trace, 7);
                if (warp < dn) {
                    const int it = i0 + warp;
                    float acc4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                    for (int qq = 0; qq < 4; ++qq)
#pragma unroll
                        for (int c2 = 0; c2 < 4; ++c2) acc4[c2] += dred[((warp * 4 + qq) * 32 + lane) * 4 + c2];
                    const int r0 = S.item_r[it], nvalid = S.item_n[it];
#pragma unroll
                    for (int e2 = 0; e2 < 2; ++e2) {
                        const int jt = 2 * (lane & 3) + e2;
                        if (jt < nvalid) {
                            const int pid = S.sp[r0 + jt];
                            const float m = pow2f(S.ashift[pid]);
                            S.ob[pid * 16 + g] = acc4[e2] * m;
                            S.ob[pid * 16 + g + 8] = acc4[2 + e2] * m;
                        }
                    }
                }
                __syncthreads();
                if (tracing && tid == 0 && u == 0 && i0 == 0) stamp(trace, 21);
            }
        }
        __syncthreads();
        if (tid < T * 16 && !S.abort) {
            const int t = tid >> 4, n = tid & 15;
            float yv = 0.0f;
            for (int jj = 0; jj < k; ++jj) yv = fmaf(S.sel_w[t * k + jj], S.ob[(t * k + jj) * 16 + n], yv);
            reinterpret_cast<__nv_bfloat16*>(p.y)[(size_t)t * H + j * 16 + n] = __float2bfloat16_rn(yv);
        }
        __syncthreads();
        off += dn_unit;
    }
    if (tracing && tid == 0) stamp(trace, 5);

    // ---- 7. never leave with copies in flight --------------------------------------------
    if (S.abort && tid == 0)
        for (int u = 0; u < ngu + ndn; ++u) mbar_wait0(mbar0 + 8 * u, p.timeout_ns);
}

}  // namespace fe
