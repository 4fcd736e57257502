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
//   1. one bulk copy brings the T router-logit rows and the T x rows into
//      shared memory; every CTA routes the T tokens itself (the rank of each
//      logit among the E logits of its token, counted by all threads in
//      parallel: rank < k selects it as slot rank, ties to the lower index)
//      and groups the T*k pairs by expert; CTA 0 also publishes the routing;
//   2. from the number of distinct routed experts every CTA reads, in a
//      table built at reserve time, its range of gate_up units (16 gate + 16
//      up columns of one routed expert) and its range of down units (16
//      output columns over all routed experts), balanced in bytes;
//   3. one thread issues cp.async.bulk copies of ALL the CTA's weight bytes
//      (both phases) into shared memory at once, one mbarrier per unit;
//   4. gate_up units: mma.m16n8k16 with the tokens of the unit's expert as
//      the N columns (mma.cuh), SiLU(gate)*up, act written to global memory
//      (L2) as 64-bit words holding the fp32 value and the launch's epoch tag;
//   5. each CTA that owns down units reads act back, polling (bounded) until
//      every word carries this launch's tag -- the data is its own ready
//      flag, so no grid-wide barrier round trip is needed;
//   6. down units: one warp per routed expert, its pairs as the N columns;
//      the 16 outputs of every pair are combined in slot order, so y is
//      written once, without atomics.
//
// The kernel is launched with programmatic dependent launch: its CTAs load
// only static data before griddepcontrol.wait, so the next layer's CTAs can
// be resident and waiting while this layer finishes.
#pragma once

#include <vector>

#include "common.cuh"
#include "mma.cuh"

namespace fe {

constexpr int kDecThreads = 512;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kDecMaxPairs = 16;   // T * top_k handled by the fused kernel
constexpr int kDecMaxItems = 48;   // weight units (mbarriers) per CTA
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
    unsigned long long* act;  // [kDecMaxPairs][I] by pair id: (epoch tag << 32) | fp32 bits
    unsigned* sync;           // [2]: CTAs that read the epoch this launch, epoch
    uint32_t* status;
    unsigned long long timeout_ns;  // bound of every wait
    uint32_t weight_bytes;    // shared memory reserved for weight units
    int bulk_inputs;          // x and logits rows copied with cp.async.bulk (16-byte aligned)
    unsigned long long* trace;  // optional [grid][16] %globaltimer stamps of the phases
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

FE_DEV unsigned ld_acquire_gpu(const unsigned* p)
{
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

FE_DEV void st_release_gpu(unsigned* p, unsigned v)
{
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

FE_DEV void st_volatile_u64(unsigned long long* p, unsigned long long v)
{
    asm volatile("st.volatile.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

FE_DEV void ld_volatile_2u64(const unsigned long long* p, unsigned long long& a, unsigned long long& b)
{
    asm volatile("ld.volatile.global.v2.u64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "l"(p) : "memory");
}

FE_DEV float logit_key(float v) { return v != v ? -INFINITY : v; }

struct DecodeShared {
    int sel_e[kDecMaxPairs];
    float sel_w[kDecMaxPairs];
    int sp[kDecMaxPairs];         // pair ids in (expert, pair) order
    int pdi[kDecMaxPairs];        // pair -> distinct-expert index
    int dex[kDecMaxPairs];        // distinct experts, ascending
    int dstart[kDecMaxPairs + 1]; // first sorted position of each distinct expert
    int plan[kDecMaxPairs + 1][4];  // per nd: gate_up first/end, down first/end of this CTA
    int xshift[kDecMaxPairs];
    int ashift[kDecMaxPairs];
    int item_d[kDecMaxPairs + 1];   // down items: (distinct expert, first sorted pair, pairs <= 8)
    int item_r[kDecMaxPairs + 1];
    int item_n[kDecMaxPairs + 1];
    int n_items;
    int nd;
    int abort;
    unsigned tag;
    float wmax[kDecWarps];
    int rank_part[kDecThreads];
    float ob[kDecMaxPairs * 16];  // down: [pair][16] outputs
};

// Byte offsets of the dynamic shared memory regions.
struct DecodeSmem {
    uint32_t mbar, shared, red, dred, xs, as, lg, xr, total;
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
    L.xs = L.red + 4u * (kDecWarps * 32 * 8 > 8 * 4 * 32 * 4 ? kDecWarps * 32 * 8 : 8 * 4 * 32 * 4);
    L.as = L.xs + 4u * (T + 1) * brow_words(H);
    L.lg = align16(L.as + 4u * (T * k + 1) * brow_words(I));
    L.xr = align16(L.lg + 4u * T * E);
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
    float* lg = reinterpret_cast<float*>(dsm + L.lg);
    uint16_t* xr = reinterpret_cast<uint16_t*>(dsm + L.xr);
    const uint32_t mbar0 = smem_addr(dsm + L.mbar);
    const uint32_t in_bar = mbar0 + 8 * kDecMaxItems;
    const bool tracing = p.trace != nullptr;
    unsigned long long* trace = tracing ? p.trace + (size_t)blockIdx.x * 16 : nullptr;
    if (tracing && tid == 0) trace[0] = globaltimer_ns();

    // ---- 0. static data only, then wait for the previous grid ---------------------
    if (tid < 4 * (kDecMaxPairs + 1)) {
        const int nd = tid >> 2, which = tid & 3;   // 0: gate_up first, 1: end, 2: down first, 3: end
        const int32_t* row = p.plan + ((size_t)nd * 2 + (which >> 1)) * (gridDim.x + 1);
        S.plan[nd][which] = row[blockIdx.x + (which & 1)];
    }
    if (tid == 0) {
        for (int u = 0; u <= kDecMaxItems; ++u) mbar_init(mbar0 + 8 * u, 1);   // the weight units' and in_bar
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        S.abort = 0;
    }
    for (int i = tid; i < xrw; i += kDecThreads) xs[T * xrw + i] = 0u;       // zero B rows
    for (int i = tid; i < arw; i += kDecThreads) as[P * arw + i] = 0u;
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (tid == 0 && p.bulk_inputs) {
        const uint32_t lb = 4u * T * E, xb = 2u * T * H;
        mbar_expect_tx(in_bar, lb + xb);
        bulk_g2s(smem_addr(lg), p.logits, lb, in_bar);
        bulk_g2s(smem_addr(xr), p.x, xb, in_bar);
    }
    // this launch's epoch (the previous launch's update is visible after
    // griddepcontrol.wait); both requests are in flight while the CTA routes and
    // their results are consumed only when act is about to be written
    unsigned ep_e0 = 0, ep_arrived = 0;
    if (tid == kDecThreads - 1) {
        ep_e0 = *reinterpret_cast<volatile unsigned*>(p.sync + 1);
        ep_arrived = atomicAdd(p.sync, 1u);
    }
    if (!p.bulk_inputs) {
        for (int i = tid; i < T * E; i += kDecThreads) lg[i] = p.logits[i];
        for (int i = tid; i < T * H; i += kDecThreads) xr[i] = p.x[i];
    }
    __syncthreads();
    if (p.bulk_inputs && !mbar_wait0(in_bar, p.timeout_ns)) {
        if (tid == 0) atomicOr(p.status, kDevLoadTimeout);
        return;
    }
    if (tracing && tid == 0) trace[8] = globaltimer_ns();

    // ---- 1. routing: rank of every logit among its token's E logits ------------------
    // nsplit threads share the comparisons of one logit (E <= 128: 2 or more)
    bool nan_seen = false;
    {
        const int epad = (E + 31) & ~31;
        const int nsplit = epad >= kDecThreads ? 1 : kDecThreads / epad;
        const int chunk = ((E + nsplit - 1) / nsplit + 3) & ~3;
        int* rk = S.rank_part;
        for (int t = 0; t < T; ++t) {
            const float* row = lg + t * E;
            for (int base = 0; base < E; base += kDecThreads / nsplit) {
                const int e = base + tid % epad, part = tid / epad;
                int rank = 0;
                if (e < E && part < nsplit) {
                    const float v = logit_key(row[e]);
                    nan_seen |= row[e] != row[e];
                    const int lo = part * chunk, hi = min(E, lo + chunk);
                    int e2 = lo;
                    if ((E & 3) == 0) {
#pragma unroll 4
                        for (; e2 + 4 <= hi; e2 += 4) {
                            const float4 o = *reinterpret_cast<const float4*>(row + e2);
                            const float o0 = logit_key(o.x), o1 = logit_key(o.y), o2 = logit_key(o.z), o3 = logit_key(o.w);
                            rank += (o0 > v) || (o0 == v && e2 < e);
                            rank += (o1 > v) || (o1 == v && e2 + 1 < e);
                            rank += (o2 > v) || (o2 == v && e2 + 2 < e);
                            rank += (o3 > v) || (o3 == v && e2 + 3 < e);
                        }
                    }
                    for (; e2 < hi; ++e2) {
                        const float o = logit_key(row[e2]);
                        rank += (o > v) || (o == v && e2 < e);
                    }
                }
                if (nsplit > 1) {
                    rk[tid] = rank;
                    __syncthreads();
                    if (part == 0 && e < E) {
                        for (int q = 1; q < nsplit; ++q) rank += rk[tid + q * epad];
                    }
                    __syncthreads();
                }
                if (part == 0 && e < E && rank < k) {
                    S.sel_e[t * k + rank] = e;
                    S.sel_w[t * k + rank] = logit_key(row[e]);
                }
            }
        }
    }
    if (tracing && tid == 0) trace[10] = globaltimer_ns();
    if (__syncthreads_or(nan_seen) && tid == 0 && blockIdx.x == 0) atomicOr(p.status, kDevNanLogit);
    for (int t = warp; t < T; t += kDecWarps) {
        const float l0 = S.sel_w[t * k];
        const float ej = lane < k ? expf(S.sel_w[t * k + lane] - l0) : 0.0f;
        const float ssum = warp_sum(ej);
        __syncwarp();
        if (lane < k) {
            const float wj = ej / ssum;
            S.sel_w[t * k + lane] = wj;
            if (blockIdx.x == 0) {
                p.idx[t * k + lane] = S.sel_e[t * k + lane];
                p.w[t * k + lane] = wj;
            }
        }
    }
    __syncthreads();

    if (tracing && tid == 0) trace[12] = globaltimer_ns();
    // ---- 2. grouping (warp 0): stable order by expert --------------------------
    if (warp == 0) {
        int ep = 0x7fffffff, rank = 0;
        if (lane < P) {
            ep = S.sel_e[lane];
            for (int q = 0; q < P; ++q) {
                const int eq = S.sel_e[q];
                rank += (eq < ep) || (eq == ep && q < lane);
            }
            S.sp[rank] = lane;
        }
        // rank r is the first pair of its expert iff no pair of the same expert has
        // a lower rank, i.e. no q < lane has the same expert
        bool first = lane < P;
        if (lane < P)
            for (int q = 0; q < lane; ++q) first &= S.sel_e[q] != ep;
        const uint32_t firsts = __ballot_sync(0xffffffffu, first);
        // distinct index of this pair's expert = distinct experts below it
        int dless = 0;
        if (lane < P)
            for (int q = 0; q < P; ++q) dless += ((firsts >> q) & 1u) && S.sel_e[q] < ep;
        if (first) {
            S.dex[dless] = ep;
            S.dstart[dless] = rank;
        }
        if (lane < P) S.pdi[lane] = dless;
        if (lane == 0) {
            S.nd = __popc(firsts);
            S.dstart[__popc(firsts)] = P;
        }
        __syncwarp();
        if (lane == 0) {
            int ni = 0;
            for (int dd = 0; dd < S.nd; ++dd)
                for (int r = S.dstart[dd]; r < S.dstart[dd + 1]; r += 8) {
                    S.item_d[ni] = dd;
                    S.item_r[ni] = r;
                    S.item_n[ni] = min(8, S.dstart[dd + 1] - r);
                    ++ni;
                }
            S.n_items = ni;
        }
        if (blockIdx.x == 0 && lane < P) {
            p.sorted_pair[lane] = S.sp[lane];
            p.pair_row[S.sp[lane]] = lane;
        }
    }
    __syncthreads();
    const int nd = S.nd;
    const int ntu = I / 16;   // gate_up units per expert
    const int gu0 = S.plan[nd][0], gu1 = S.plan[nd][1], dn0 = S.plan[nd][2], dn1 = S.plan[nd][3];
    const int ngu = gu1 - gu0, ndn = dn1 - dn0;
    const uint32_t dn_unit = (uint32_t)nd * dn_blk;
    if (tracing && tid == 0) trace[9] = globaltimer_ns();

    // ---- 3. warp 0 issues every weight load of this CTA now -------------------------
    if (warp == 0) {
        if (lane == 0) {
            for (int u = 0; u < ngu; ++u) mbar_expect_tx(mbar0 + 8 * u, gu_unit);
            for (int u = 0; u < ndn; ++u) mbar_expect_tx(mbar0 + 8 * (ngu + u), dn_unit);
        }
        __syncwarp();
        const uint32_t wb = smem_addr(wbuf);
        for (int u = lane; u < ngu; u += 32) {
            const int gid = gu0 + u, dd = gid / ntu, j = gid - dd * ntu;
            bulk_g2s(wb + u * gu_unit, p.gu_blocks + ((size_t)S.dex[dd] * ntu + j) * gu_unit, gu_unit, mbar0 + 8 * u);
        }
        for (int i = lane; i < ndn * nd; i += 32) {
            const int u = i / nd, dd = i - u * nd, j = dn0 + u;
            bulk_g2s(wb + ngu * gu_unit + u * dn_unit + dd * dn_blk,
                     p.dn_blocks + ((size_t)S.dex[dd] * (H / 16) + j) * dn_blk, dn_blk, mbar0 + 8 * (ngu + u));
        }
        if (tracing && lane == 0) trace[1] = globaltimer_ns();
    }
    if (blockIdx.x == 0) {
        for (int e = tid; e <= E; e += kDecThreads) {
            int below = 0, eq = 0;
            for (int q = 0; q < P; ++q) {
                below += S.sel_e[q] < e;
                eq += S.sel_e[q] == e;
            }
            p.offsets[e] = below;
            if (e < E) p.counts[e] = eq;
        }
    }

    // ---- 4. x rows as fp16 pairs with a power-of-two shift per token (whole CTA) -------
    for (int t = 0; t < T; ++t) {
        const uint32_t* xw = reinterpret_cast<const uint32_t*>(xr + (size_t)t * H);
        float m = 0.0f;
        for (int r = tid; r < H / 2; r += kDecThreads) {
            const uint32_t two = xw[r];
            m = fmaxf(m, fmaxf(fabsf(bf16_bits_to_f32((uint16_t)(two & 0xffff))),
                               fabsf(bf16_bits_to_f32((uint16_t)(two >> 16)))));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) S.wmax[warp] = m;
        __syncthreads();
        float mm = 0.0f;
#pragma unroll
        for (int w2 = 0; w2 < kDecWarps; ++w2) mm = fmaxf(mm, S.wmax[w2]);
        const int sh = fp16_shift(mm);
        const float scl = pow2f(-sh);
        if (tid == 0) S.xshift[t] = sh;
        for (int r = tid; r < H / 2; r += kDecThreads) {
            const uint32_t two = xw[r];
            xs[t * xrw + r] = f32x2_to_f16x2_rn(bf16_bits_to_f32((uint16_t)(two & 0xffff)) * scl,
                                               bf16_bits_to_f32((uint16_t)(two >> 16)) * scl);
        }
        __syncthreads();
    }
    if (tracing && tid == 0) trace[2] = globaltimer_ns();

    if (tid == kDecThreads - 1) {
        const unsigned tg = (ep_e0 + 1u) ? (ep_e0 + 1u) : 1u;
        S.tag = tg;
        if (ep_arrived == gridDim.x - 1) {
            // every CTA has read the epoch: advance it for the next launch
            atomicExch(p.sync, 0u);
            st_release_gpu(p.sync + 1, tg);
        }
    }
    __syncthreads();

    // ---- 5. gate_up units -> tagged act ------------------------------------------------
    uint32_t off = 0;
    for (int u = 0; u < ngu; ++u) {
        const uint32_t bar = mbar0 + 8 * u;
        if (!mbar_wait0(bar, p.timeout_ns)) {
            if (tid == 0) { atomicOr(p.status, kDevLoadTimeout); S.abort = 1; }
        }
        __syncthreads();
        if (S.abort) break;
        const int gid = gu0 + u, dd = gid / ntu, j = gid - dd * ntu;
        const uint8_t* blk0 = wbuf + off;
        const uint8_t* blk1 = blk0 + block_bytes(H);
        const int r0 = S.dstart[dd], r1 = S.dstart[dd + 1];
        for (int nb = r0; nb < r1; nb += 8) {
            const int nvalid = min(8, r1 - nb);
            const uint32_t* brow = xs + (g < nvalid ? S.sp[nb + g] / k : T) * xrw;
            float t0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, t1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            for (int q = warp; q < H / 64; q += kDecWarps) quad_mma2(blk0, blk1, H, brow, q, lane, t0, t1);
            float* rl = red + (warp * 32 + lane) * 8;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                rl[i] = t0[i];
                rl[4 + i] = t1[i];
            }
            __syncthreads();
            if (tid < 128) {
                const int n = tid & 15, jt = tid >> 4;
                if (jt < nvalid) {
                    const int ln = 4 * (n & 7) + (jt >> 1), idx = (n >> 3) * 2 + (jt & 1);
                    float gs = 0.0f, us = 0.0f;
#pragma unroll
                    for (int w2 = 0; w2 < kDecWarps; ++w2) {
                        gs += red[(w2 * 32 + ln) * 8 + idx];
                        us += red[(w2 * 32 + ln) * 8 + 4 + idx];
                    }
                    const int pid = S.sp[nb + jt], t = pid / k;
                    const float m = pow2f(S.xshift[t]);
                    const float a = silu_mul(gs * m, us * m);
                    st_volatile_u64(p.act + (size_t)pid * I + 16 * j + n, ((unsigned long long)S.tag << 32) | __float_as_uint(a));
                }
            }
            __syncthreads();
        }
        off += gu_unit;
    }
    if (tracing && tid == 0) trace[3] = globaltimer_ns();

    // ---- 6. down units: read act back (tagged), compute, combine ------------------------
    const unsigned tag = S.tag;
    if (ndn > 0 && !S.abort) {
        // warp pp stages pair pp: up to 16 chunks of two tagged words per lane, all
        // requested at once, then only the late ones again
        for (int pp = warp; pp < P; pp += kDecWarps) {
            const unsigned long long* src = p.act + (size_t)pp * I;
            unsigned long long a0[16], a1[16];
            uint32_t pending = 0;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int r = lane + 32 * i;
                a0[i] = a1[i] = 0ull;
                if (2 * r < I) {
                    ld_volatile_2u64(src + 2 * r, a0[i], a1[i]);
                    if ((unsigned)(a0[i] >> 32) != tag || (unsigned)(a1[i] >> 32) != tag) pending |= 1u << i;
                }
            }
            if (__any_sync(0xffffffffu, pending != 0)) {
                const unsigned long long t0 = globaltimer_ns();
                bool late = false;
                while (__any_sync(0xffffffffu, pending != 0) && !late) {
                    __nanosleep(100);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        if ((pending >> i) & 1u) {
                            ld_volatile_2u64(src + 2 * (lane + 32 * i), a0[i], a1[i]);
                            if ((unsigned)(a0[i] >> 32) == tag && (unsigned)(a1[i] >> 32) == tag) pending &= ~(1u << i);
                        }
                    }
                    late = __any_sync(0xffffffffu, globaltimer_ns() - t0 > p.timeout_ns);
                }
                if (late && lane == 0) {
                    atomicOr(p.status, kDevBarrierTimeout);
                    S.abort = 1;
                }
            }
            float m = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i)
                m = fmaxf(m, fmaxf(fabsf(__uint_as_float((uint32_t)a0[i])), fabsf(__uint_as_float((uint32_t)a1[i]))));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            const int sh = fp16_shift(m);
            const float scl = pow2f(-sh);
            if (lane == 0) S.ashift[pp] = sh;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int r = lane + 32 * i;
                if (2 * r < I)
                    as[pp * arw + r] = f32x2_to_f16x2_rn(__uint_as_float((uint32_t)a0[i]) * scl,
                                                        __uint_as_float((uint32_t)a1[i]) * scl);
            }
        }
        __syncthreads();
    }
    if (tracing && tid == 0) trace[4] = globaltimer_ns();
    for (int u = 0; u < ndn; ++u) {
        const uint32_t bar = mbar0 + 8 * (ngu + u);
        if (!mbar_wait0(bar, p.timeout_ns)) {
            if (tid == 0) { atomicOr(p.status, kDevLoadTimeout); S.abort = 1; }
        }
        __syncthreads();
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
                for (int q = qa; q < qb; ++q) {
#pragma unroll
                    for (int m = 0; m < TPW; ++m) {
                        const int i = (warp >> 2) + (kDecWarps / 4) * m;
                        if (i < dn) {
                            const int it = i0 + i;
                            const int r0 = S.item_r[it], nvalid = S.item_n[it];
                            const uint32_t* brow = as + (g < nvalid ? S.sp[r0 + g] : P) * arw;
                            quad_mma(wbuf + off + S.item_d[it] * dn_blk, I, brow, q, lane, tot[m]);
                        }
                    }
                }
#pragma unroll
                for (int m = 0; m < TPW; ++m) {
                    const int i = (warp >> 2) + (kDecWarps / 4) * m;
                    if (i < dn)
#pragma unroll
                        for (int c2 = 0; c2 < 4; ++c2) dred[((i * 4 + quarter) * 32 + lane) * 4 + c2] = tot[m][c2];
                }
                __syncthreads();
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
    if (tracing && tid == 0) trace[5] = globaltimer_ns();

    // ---- 7. never leave with copies in flight --------------------------------------------
    if (S.abort && tid == 0)
        for (int u = 0; u < ngu + ndn; ++u) mbar_wait0(mbar0 + 8 * u, p.timeout_ns);
}

}  // namespace fe
