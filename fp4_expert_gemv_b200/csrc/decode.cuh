// Fused small-T decode layer: one launch per layer, the expert MLPs split over
// the CTAs along the intermediate dimension.
//
// "FireEcho Engine", sections "Speed Optimization History" (single-token
// decode fast path, multi-expert kernel, packed contiguous expert buffer,
// CUDA-graph decode) and "The Goliath Kernel: Why It's Fast" (expert IDs read
// on the GPU, FP4 dequantised in registers, tensor-core accumulation, nothing
// dequantised written to memory).  The pages' kernel runs one Triton launch
// per projection; here the whole layer is one launch and each CTA owns whole
// slices of the routed experts' MLPs:
//
//   1. every CTA routes the T tokens itself (one warp per token: warp top-k
//      over orderable keys, ties to the lower index, softmax over the k
//      selected) and groups the T*k pairs by expert; CTA 0 publishes the
//      routing; a bulk copy brings the x rows into shared memory meanwhile;
//   2. the nd routed experts' act columns form U = nd * I/16 units of 16
//      columns; CTA c takes units [c U / G, (c+1) U / G) of the expert-major
//      sequence (G = grid).  A unit's weights are its gate_up pair of blocks
//      (16 gate + 16 up columns over K = H, 18H bytes) and the 16 matching
//      rows of W_dn over all H outputs (8H bytes of codes + the row group's
//      2H bytes of scales, shared by the two units of a 32-row group); one
//      warp issues a cp.async.bulk copy of each into shared memory as soon as
//      the routing is known, one mbarrier per copy;
//   3. per unit, as its bytes land: gate_up on the tensor cores (mma.m16n8k16,
//      E2M1 codes turned into f16 in registers, the unit expert's tokens as
//      the N columns, x fragments held in registers), a reduction over the
//      warps and SiLU(gate) * up -- act never leaves the CTA; the 16 act
//      values of each token times the token's slot weight become the B
//      operand (one column per token) of the down product, and every warp adds
//      the unit's contribution to its share of the H outputs in registers (the
//      16 rows of W_dn are the K of one mma per 16 outputs);
//   4. the CTA's partial y (T x H, fp32) goes to its own slot in global
//      memory, then the CTA arrives on a counter (release); CTA c < H/16 waits
//      (acquire) for every CTA of the launch and sums the output columns
//      [16c, 16c + 16) over the CTAs in a fixed order, so y is written once,
//      bit-reproducibly, with no atomic on data.
//
// Every wait is bounded by %globaltimer.  The counter wait needs every CTA of
// the launch resident at once (grid = number of SMs, one CTA per SM), which
// the host checks from the kernel's occupancy before it takes this path.  The
// kernel is launched with programmatic dependent launch: before
// griddepcontrol.wait its CTAs set up only static state (and ask L2 for the
// logits and x rows, which is safe: an L2 prefetch fills no L1 line).
#pragma once

#include "bulk.cuh"
#include "common.cuh"
#include "mma.cuh"
#include "warp_route.cuh"

namespace fe {

constexpr int kDecThreads = 512;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kDecMaxPairs = 16;      // T * top_k handled by the fused kernel
constexpr int kDecMaxT = 8;           // tokens: one 8-column block of the mma
constexpr int kDecMaxUnits = 4;       // units (16 act columns of one expert) per CTA
constexpr int kDecMaxE = 512;         // experts routed by one warp: 16 logits per lane
constexpr int kDecMaxH = 2048;        // outputs: 2 quads of 64 columns per warp, in registers
constexpr int kDecHQuadsPerWarp = kDecMaxH / 64 / kDecWarps;
constexpr int kDecCandCap = 128;      // candidate keys per routing warp (in the partials' space)
constexpr int kDecRedFloats = 4096;   // gate_up partials of a unit; routing candidates; final sums
constexpr int kDecSlots = kDecThreads / 16;   // partial-sum slots of the final column reduction
constexpr int kDecMaxCtas = 160;      // grid (= SMs) the final reduction is unrolled for
constexpr int kDecArriveSlack = 8;    // CTAs still out when the column sums start reading
constexpr uint32_t kDevBarrierTimeout = 0x4;
constexpr uint32_t kDevLoadTimeout = 0x8;

struct DecodeParams {
    const uint16_t* x;        // bf16 [T][H]
    const float* logits;      // [T][E]
    uint16_t* y;              // bf16 [T][H]
    int T, E, H, I, k;
    const uint8_t* gu_blocks; // [E][I/16] gate_up units of 2 blocks (18H bytes)
    const uint8_t* dn_rows;   // [E][I/32] row groups of W_dn (18H bytes, pack.cuh)
    const uint8_t* fmt;       // [E]: 1 = the expert's weights are INT2 codes (below); null: all E2M1
    const uint8_t* gu2_blocks;  // INT2 experts: [E][I/16] gate_up units of 2 INT2 blocks (10H bytes)
    const uint8_t* dn2_rows;    // INT2 experts: [E][I/32] INT2 row groups of W_dn (10H bytes)
    int32_t* idx;
    float* w;
    int32_t* counts;
    int32_t* offsets;
    int32_t* sorted_pair;
    int32_t* pair_row;
    unsigned long long* part; // [grid][T][H] per-CTA partial outputs: (launch tag << 32) | fp32 bits
    unsigned long long* epoch;  // [grid + 1]: launches CTA c has run on this handle; [grid]: arrivals
    uint32_t* status;
    unsigned long long timeout_ns;  // bound of every wait on copies
    unsigned long long exchange_timeout_ns;  // bound of the wait for the other CTAs' arrivals
    int extra_arrivals;       // tests only: 1 = the column sums wait for a launch more than this one (never)
    uint32_t weight_bytes;    // shared memory reserved for weight units
    int bulk_inputs;          // x rows copied with cp.async.bulk (16-byte aligned)
    unsigned long long* trace;  // optional [grid][64]: %globaltimer (0-31) and clock64 (32-63) stamps
};

// Units of one layer and the range of CTA c (all integer, the same on the host).
__host__ __device__ inline int dec_units(int nd, int I) { return nd * (I / 16); }
// (32-bit arithmetic: c <= kDecMaxCtas and U <= kDecMaxPairs * 64, so c * U < 2^32)
__host__ __device__ inline int dec_unit_first(int c, int U, int G) { return (int)((unsigned)c * (unsigned)U / (unsigned)G); }
// Shared memory a CTA's units need at most: gate_up 18H + down 10H each.
__host__ __device__ inline uint32_t dec_unit_bytes(int H) { return 28u * (uint32_t)H; }

struct DecodeShared {
    int sel_e[kDecMaxPairs];
    float sel_w[kDecMaxPairs];
    int sp[kDecMaxPairs];         // pair ids in (expert, pair) order
    int pdi[kDecMaxPairs];        // pair -> distinct-expert index
    int dex[kDecMaxPairs];        // distinct experts, ascending
    int dstart[kDecMaxPairs + 1]; // first sorted position of each distinct expert
    int xshift[kDecMaxT];
    int nd;
    int abort;
    int u0, nu;                               // this CTA's units
    uint32_t u_codes[kDecMaxUnits];           // shared-memory offsets of a unit's down codes
    uint32_t u_scales[kDecMaxUnits];          // ... and of its row group's scales
    int u_dnbar[kDecMaxUnits];                // barrier of its down copy
    int u_fmt[kDecMaxUnits];                  // 1: the unit's expert is INT2
    uint32_t dn_bytes[kDecMaxUnits];          // bytes of the down copy a unit issued (0: shares one)
    int bshift[kDecMaxT];                     // current unit: power-of-two shift of each token's B column
    uint32_t bfrag[kDecMaxT][8];              // current unit's down B operand: token t, 16 values as f16x2
    unsigned long long target;                // arrivals that complete this launch
    unsigned tag;                             // this launch's tag of the partial words
    float wmax[2][kDecWarps];
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
    }
    if (lane == 0) {
        S.nd = k;
        S.dstart[k] = k;
    }
    __syncwarp();
}

// Several tokens: stable order of the P <= 32 pairs by expert, by one warp.
FE_DEV void group_tokens(DecodeShared& S, int P, int lane)
{
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
    if (lane < P) {
        S.sp[rank] = lane;
        S.pdi[lane] = dless;
    }
    if (first) {
        S.dex[dless] = ep;
        S.dstart[dless] = rank;
    }
    if (lane == 0) {
        S.nd = __popc(firsts);
        S.dstart[__popc(firsts)] = P;
    }
    __syncwarp();
}

// Byte offsets of the dynamic shared memory regions.
struct DecodeSmem {
    uint32_t mbar, shared, red, xs, xr, total;
};

__host__ __device__ inline uint32_t align16(uint32_t v) { return (v + 15u) & ~15u; }

// weights | mbarriers (gate_up, down, x) | DecodeShared | red | xs: T x rows
// + 1 zero row (brow_words each) | xr: raw x rows
__host__ __device__ inline DecodeSmem decode_smem_layout(uint32_t weight_bytes, int T, int H)
{
    DecodeSmem L;
    L.mbar = weight_bytes;
    L.shared = L.mbar + 8 * (2 * kDecMaxUnits + 1);
    L.red = align16(L.shared + (uint32_t)sizeof(DecodeShared));
    static_assert(kDecRedFloats * 4 >= kDecWarps * kDecCandCap * 8, "routing candidates space");
    static_assert(kDecRedFloats >= kDecWarps * kDecMaxT * 32, "gate_up partials space");
    static_assert(kDecRedFloats >= kDecMaxT * kDecSlots * 16, "final sums space");
    L.xs = L.red + 4u * kDecRedFloats;
    L.xr = align16(L.xs + 4u * (T + 1) * brow_words(H));
    L.total = align16(L.xr + 2u * T * H);
    return L;
}

__global__ void __launch_bounds__(kDecThreads, 1) decode_kernel(DecodeParams p)
{
    extern __shared__ __align__(128) uint8_t dsm[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, c4 = lane & 3;
    const int T = p.T, E = p.E, H = p.H, I = p.I, k = p.k, P = T * k;
    const int G = gridDim.x;
    const DecodeSmem L = decode_smem_layout(p.weight_bytes, T, H);
    const uint32_t gu_unit = 2u * block_bytes(H);
    const int xrw = brow_words(H);
    const int upe = I / 16;   // units per expert

    uint8_t* wbuf = dsm;
    DecodeShared& S = *reinterpret_cast<DecodeShared*>(dsm + L.shared);
    float* red = reinterpret_cast<float*>(dsm + L.red);
    uint32_t* xs = reinterpret_cast<uint32_t*>(dsm + L.xs);
    uint16_t* xr = reinterpret_cast<uint16_t*>(dsm + L.xr);
    const uint32_t mbar0 = smem_addr(dsm + L.mbar);   // [0, 4): gate_up, [4, 8): down, 8: x
    const uint32_t in_bar = mbar0 + 8 * (2 * kDecMaxUnits);
    auto bar_gu = [&](int i) { return mbar0 + 8u * (uint32_t)i; };
    auto bar_dn = [&](int i) { return mbar0 + 8u * (uint32_t)(kDecMaxUnits + i); };
    const bool tracing = p.trace != nullptr;
    unsigned long long* trace = tracing ? p.trace + (size_t)blockIdx.x * 64 : nullptr;
    if (tracing && tid == 0) stamp(trace, 0);

    // ---- 0. static state only, then wait for the previous grid ---------------------
    if (warp == 1) {
        for (int u = lane; u <= 2 * kDecMaxUnits; u += 32) mbar_init(mbar0 + 8 * u, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        if (lane == 0) S.abort = 0;
    }
    for (int i = tid; i < xrw; i += kDecThreads) xs[T * xrw + i] = 0u;   // the zero B row
    if (tid < kDecMaxT * 8) S.bfrag[tid >> 3][tid & 7] = 0u;             // tokens past T: zero columns
    if (tid < kDecMaxT) S.bshift[tid] = 0;
    // the logits and x rows into L2 while the previous grid finishes: an L2
    // prefetch fills no L1 line, and a write of the previous grid lands in L2,
    // so what is read after the wait is current either way
    if (warp == 2) {
        const char* lb = reinterpret_cast<const char*>(p.logits);
        for (int o = lane * 128; o < T * E * 4; o += 32 * 128) prefetch_l2(lb + o);
        const char* xb = reinterpret_cast<const char*>(p.x);
        for (int o = lane * 128; o < T * H * 2; o += 32 * 128) prefetch_l2(xb + o);
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (tracing && tid == 0) {
        stamp(trace, 8);
        // diagnostics: the latency of the logits row alone (the routing then finds it in L1)
        const float lv = *reinterpret_cast<const volatile float*>(p.logits);
        if (lv == 12345.0f) trace[63] = 1;
        stamp(trace, 27);
    }
    if (warp == 1 && lane == 16 && p.bulk_inputs) {
        const uint32_t xb = 2u * T * H;
        mbar_expect_tx(in_bar, xb);
        bulk_g2s(smem_addr(xr), p.x, xb, in_bar);
    }
    // this launch's arrival target: every launch runs every CTA (the grid is
    // fixed per handle) and each CTA arrives once, so the per-CTA launch counts
    // move in lockstep and all CTAs derive the same target
    unsigned long long ep_e0 = 0;
    if (tid == kDecThreads - 1) ep_e0 = *reinterpret_cast<volatile unsigned long long*>(p.epoch + blockIdx.x);
    const int nroute = min(T, kDecWarps);
    const int cap = (kDecWarps * kDecCandCap) / nroute;
    unsigned long long* cand = reinterpret_cast<unsigned long long*>(red) + warp * cap;

    // ---- 1. routing: warp t selects the top-k logits of token t ----------------------
    // With T = 1, warp 0 routes and hands the selection to warp 1, which groups
    // and issues the copies; the softmax comes after.  With T > 1 every token's
    // warp also takes its softmax, then the CTA meets before the grouping.
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

    if (warp == 1) {
        // ---- 2. grouping, then this CTA's units and every one of their copies --------
        if (T == 1) {
            asm volatile("bar.sync 3, 64;" ::: "memory");
            group_single_token(S, k, lane);
        } else {
            group_tokens(S, P, lane);
        }
        if (tracing && lane == 0) stamp(trace, 9);
        // the staging warps were parked until now, so that the path to the copies
        // had the SM to itself
        asm volatile("bar.arrive 2, %0;" ::"n"(kDecThreads - 32) : "memory");
        const int U = dec_units(S.nd, I);
        const int u0 = dec_unit_first(blockIdx.x, U, G), nu = dec_unit_first(blockIdx.x + 1, U, G) - u0;
        if (lane == 0) {
            S.u0 = u0;
            S.nu = nu;
        }
        // lane i < nu plans and issues unit i's two copies.  Down regions follow the
        // gate_up slots in unit order; two units of one 32-row group in this CTA (an
        // even row block followed by the odd one) share one copy of the group
        // (codes, scales, codes), which the first of them issues.
        const int u = u0 + lane, d = u / upe, j = u - d * upe;
        const int d_next = __shfl_down_sync(0xffffffffu, d, 1), d_prev = __shfl_up_sync(0xffffffffu, d, 1);
        const bool mine = lane < nu;
        const bool first = mine && (j & 1) == 0 && lane + 1 < nu && d_next == d;
        const bool second = mine && (j & 1) == 1 && lane > 0 && d_prev == d;
        // an INT2 expert (fmt) has half the code bytes: 4H per 16 rows of W_dn, 5H per
        // gate_up block; its row groups and units come from the INT2 buffers
        const bool i2 = mine && p.fmt != nullptr && p.fmt[S.dex[d]] != 0;
        const uint32_t CH = i2 ? 4u * H : 8u * H, SH = 2u * H;   // codes of 16 rows; scales of 32
        const uint32_t dn_bytes = !mine || second ? 0u : first ? 2u * CH + SH : CH + SH;
        const uint32_t gu_bytes = i2 ? 2u * int2_block_bytes(H) : gu_unit;
        uint32_t incl = dn_bytes;   // inclusive scan of the down bytes over the lanes
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        const uint32_t off = (uint32_t)nu * gu_unit + incl - dn_bytes;
        const uint32_t off_prev = __shfl_up_sync(0xffffffffu, off, 1);   // a pair's first unit
        const long long grp = mine ? ((long long)S.dex[d] * (I / 32) + j / 2) * (long long)(2u * CH + SH) : 0ll;
        if (mine) {
            uint32_t codes, scales;
            if (second) {
                codes = off_prev + CH + SH;
                scales = off_prev + CH;
            } else if ((j & 1) == 0) {
                codes = off;
                scales = off + CH;
            } else {
                codes = off + SH;
                scales = off;
            }
            S.u_codes[lane] = codes;
            S.u_scales[lane] = scales;
            S.u_dnbar[lane] = second ? lane - 1 : lane;
            S.u_fmt[lane] = i2 ? 1 : 0;
            S.dn_bytes[lane] = dn_bytes;
            mbar_expect_tx(bar_gu(lane), gu_bytes);
            if (dn_bytes) mbar_expect_tx(bar_dn(lane), dn_bytes);
        }
        if (tracing && lane == 0) stamp(trace, 15);
        if (mine) {
            const uint32_t wb = smem_addr(wbuf);
            const uint8_t* gsrc = i2 ? p.gu2_blocks : p.gu_blocks;
            const uint8_t* dsrc = i2 ? p.dn2_rows : p.dn_rows;
            bulk_g2s(wb + lane * gu_unit, gsrc + ((size_t)S.dex[d] * upe + j) * gu_bytes, gu_bytes, bar_gu(lane));
            if (dn_bytes) bulk_g2s(wb + off, dsrc + grp + ((j & 1) && !first ? CH : 0u), dn_bytes, bar_dn(lane));
        }
        if (tracing && lane == 0) stamp(trace, 1);
    } else if (warp == 0) {
        // ---- the routing's remaining outputs; the next layer's prefetch ------------------
        if (T == 1) warp_softmax(S.sel_w, k, lane);
        if (blockIdx.x == 0) {
            for (int q = lane; q < P; q += 32) {
                p.idx[q] = S.sel_e[q];
                p.w[q] = S.sel_w[q];
            }
        }
    } else {
        asm volatile("bar.sync 2, %0;" ::"n"(kDecThreads - 32) : "memory");
        // ---- (warps 2..) x rows as fp16 pairs with a power-of-two shift per token -----
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
            S.target = (ep_e0 + 1ull) * (unsigned long long)G;
            S.tag = (unsigned)((ep_e0 + 1ull) % 0xffffffffull) + 1u;   // never 0 (the buffer's first contents)
            p.epoch[blockIdx.x] = ep_e0 + 1ull;
        }
    }
    __syncthreads();

    // ---- 3. the units: gate_up + SwiGLU, then the down contribution ---------------------
    const int nu = S.nu, u0 = S.u0;
    const int nq = H / 64;              // 64-k quads of gate_up (K = H); 64-column quads of down
    constexpr int HQ = kDecHQuadsPerWarp;
    float Y[HQ][4][4];                  // down sums: [quad slot][tile][fragment], outputs of this warp
#pragma unroll
    for (int a = 0; a < HQ; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b)
#pragma unroll
            for (int c = 0; c < 4; ++c) Y[a][b][c] = 0.0f;
    for (int i = 0; i < nu; ++i) {
        const int u = u0 + i, d = u / upe;
        if (*reinterpret_cast<volatile int*>(&S.abort) == 0 && !mbar_wait0(bar_gu(i), p.timeout_ns)) {
            atomicOr(p.status, kDevLoadTimeout);
            S.abort = 1;
        }
        if (tracing && tid == 0 && (i == 0 || i == nu - 1)) stamp(trace, i == 0 ? 11 : 13);
        const bool ui2 = S.u_fmt[i] != 0;   // the same in every thread
        const uint8_t* blk0 = wbuf + i * gu_unit;
        const uint8_t* blk1 = blk0 + (ui2 ? int2_block_bytes(H) : block_bytes(H));
        const int r0 = S.dstart[d], nvalid = S.dstart[d + 1] - r0;   // the expert's tokens (<= T <= 8)
        const uint32_t* brow = xs + (g < nvalid ? S.sp[r0 + g] / k : T) * xrw;
        float t0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, t1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        // warp w takes the 64-k quads w, w + W, ...: one compact loop (the code of a
        // launch is fetched cold, so a short loop body beats unrolled copies), the
        // quad's x fragments read from shared memory with two 16-byte loads
        if (ui2) {
#pragma unroll 1
            for (int q = warp; q < nq; q += kDecWarps) {
                uint32_t b[8];
                load_bfrag(brow, q, lane, b);
                quad_mma2_b_int2(blk0, blk1, H, b, q, lane, t0, t1);
            }
        } else {
#pragma unroll 1
            for (int q = warp; q < nq; q += kDecWarps) {
                uint32_t b[8];
                load_bfrag(brow, q, lane, b);
                quad_mma2_b(blk0, blk1, H, b, q, lane, t0, t1);
            }
        }
        if (tracing && tid == 0 && i == nu - 1) stamp(trace, 17);
        // partials of the valid token columns: [warp][column][gate 16 | up 16];
        // lane (g, c) holds rows g, g+8 of columns 2c, 2c+1
        {
            float* rw = red + warp * nvalid * 32;
            if (2 * c4 < nvalid) {
                rw[(2 * c4) * 32 + g] = t0[0];
                rw[(2 * c4) * 32 + g + 8] = t0[2];
                rw[(2 * c4) * 32 + 16 + g] = t1[0];
                rw[(2 * c4) * 32 + 24 + g] = t1[2];
            }
            if (2 * c4 + 1 < nvalid) {
                rw[(2 * c4 + 1) * 32 + g] = t0[1];
                rw[(2 * c4 + 1) * 32 + g + 8] = t0[3];
                rw[(2 * c4 + 1) * 32 + 16 + g] = t1[1];
                rw[(2 * c4 + 1) * 32 + 24 + g] = t1[3];
            }
        }
        __syncthreads();
        // act of column n (warp n): the 8 warps' partials summed, SiLU(gate) * up,
        // times the pair's slot weight; its 16 values become token t's B column
        // (f16 with a power-of-two shift), tokens of other experts get zeros
        if (warp < nvalid) {
            const int half = lane >> 4, cc = lane & 15;
            float s = 0.0f;
#pragma unroll
            for (int w2 = 0; w2 < kDecWarps; ++w2) s += red[(w2 * nvalid + warp) * 32 + half * 16 + cc];
            const float other = __shfl_xor_sync(0xffffffffu, s, 16);
            const int pid = S.sp[r0 + warp], t = pid / k;
            const float m = pow2f(S.xshift[t]);
            const float v = half == 0 ? silu_mul_fast(s * m, other * m) * S.sel_w[pid] : 0.0f;
            // the row max: non-negative floats order as their bits, so one warp reduction
            // (the other half-warp holds zeros)
            const float mx = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(v))));
            const int sh = fp16_shift(mx);
            const float sc = pow2f(-sh);
            const float vn = __shfl_down_sync(0xffffffffu, v, 1);
            if (half == 0 && (cc & 1) == 0) S.bfrag[t][cc >> 1] = f32x2_to_f16x2_rn(v * sc, vn * sc);
            if (lane == 0) S.bshift[t] = sh;
        } else if (warp == kDecWarps - 1 && T > 1) {
            // tokens without a pair on this expert: zero columns
            for (int l = lane; l < T * 8; l += 32) {
                const int t = l >> 3;
                bool has = false;
                for (int q = 0; q < nvalid; ++q) has |= S.sp[r0 + q] / k == t;
                if (!has) S.bfrag[t][l & 7] = 0u;
            }
        }
        __syncthreads();
        if (tracing && tid == 0 && i == nu - 1) stamp(trace, 18);
        if (*reinterpret_cast<volatile int*>(&S.abort) == 0 && !mbar_wait0(bar_dn(S.u_dnbar[i]), p.timeout_ns)) {
            atomicOr(p.status, kDevLoadTimeout);
            S.abort = 1;
        }
        if (*reinterpret_cast<volatile int*>(&S.abort) == 0) {
            // down: warp w takes output quads w, w + 8, ... (4 tiles of 16 outputs each);
            // one mma per tile with the unit's 16 rows of W_dn as K and the tokens as N
            const uint32_t b0 = S.bfrag[g][c4], b1 = S.bfrag[g][c4 + 4];
            const float m0 = pow2f(S.bshift[2 * c4]), m1 = pow2f(S.bshift[2 * c4 + 1]);
            const uint8_t* codes = wbuf + S.u_codes[i];
            const uint8_t* scl = wbuf + S.u_scales[i];
            // an INT2 register holds twice the level: the scale is halved
            if (ui2) {
#pragma unroll
                for (int qs = 0; qs < HQ; ++qs) {
                    const int q = warp + kDecWarps * qs;
                    if (q < nq) {
                        const uint2 cw = *reinterpret_cast<const uint2*>(codes + 256 * q + 8 * lane);
#pragma unroll
                        for (int h2 = 0; h2 < 2; ++h2) {   // word h2: column tiles 2 h2, 2 h2 + 1
                            uint32_t ar[8];
                            int2x8_to_f16x2x8(h2 ? cw.y : cw.x, ar);
#pragma unroll
                            for (int sl = 0; sl < 2; ++sl) {
                                const int s4 = 2 * h2 + sl;
                                const uint32_t a[4] = {ar[4 * sl], ar[4 * sl + 1], ar[4 * sl + 2], ar[4 * sl + 3]};
                                float dd[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                                mma16816(dd, a, b0, b1);
                                const uint32_t sw = *reinterpret_cast<const uint32_t*>(scl + 32 * (4 * q + s4) + 4 * g);
                                const float slo = __uint_as_float(sw << 16) * 0.5f;
                                const float shi = __uint_as_float(sw & 0xffff0000u) * 0.5f;
                                Y[qs][s4][0] = fmaf(dd[0], slo * m0, Y[qs][s4][0]);
                                Y[qs][s4][1] = fmaf(dd[1], slo * m1, Y[qs][s4][1]);
                                Y[qs][s4][2] = fmaf(dd[2], shi * m0, Y[qs][s4][2]);
                                Y[qs][s4][3] = fmaf(dd[3], shi * m1, Y[qs][s4][3]);
                            }
                        }
                    }
                }
            } else {
#pragma unroll
                for (int qs = 0; qs < HQ; ++qs) {
                    const int q = warp + kDecWarps * qs;
                    if (q < nq) {
                        const uint4 cw = *reinterpret_cast<const uint4*>(codes + 512 * q + 16 * lane);
                        const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
                        for (int s4 = 0; s4 < 4; ++s4) {
                            uint32_t a[4];
                            e2m1x8_to_f16x2x4(words[s4], a);
                            float dd[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                            mma16816(dd, a, b0, b1);
                            const uint32_t sw = *reinterpret_cast<const uint32_t*>(scl + 32 * (4 * q + s4) + 4 * g);
                            const float slo = __uint_as_float(sw << 16), shi = __uint_as_float(sw & 0xffff0000u);
                            Y[qs][s4][0] = fmaf(dd[0], slo * m0, Y[qs][s4][0]);
                            Y[qs][s4][1] = fmaf(dd[1], slo * m1, Y[qs][s4][1]);
                            Y[qs][s4][2] = fmaf(dd[2], shi * m0, Y[qs][s4][2]);
                            Y[qs][s4][3] = fmaf(dd[3], shi * m1, Y[qs][s4][3]);
                        }
                    }
                }
            }
        }
    }
    if (tracing && tid == 0) stamp(trace, 3);

    // ---- 4. this CTA's partial y (zeros for a CTA without units), then one arrival ------
    // Each value goes out as one 64-bit word with this launch's tag (single-copy
    // atomic: a reader sees the old tag or the new value), so the words are their
    // own ready flags and need no fence; the arrival counter only tells the CTAs
    // that sum the columns when to start reading.
    if (!S.abort) {
        unsigned long long* part = p.part + (size_t)blockIdx.x * T * H;
        const unsigned long long tg = (unsigned long long)S.tag << 32;
#pragma unroll
        for (int qs = 0; qs < HQ; ++qs) {
            const int q = warp + kDecWarps * qs;
            if (q < nq) {
#pragma unroll
                for (int s4 = 0; s4 < 4; ++s4) {
                    const int h0 = 16 * (4 * q + s4) + g;
                    if (2 * c4 < T) {
                        st_relaxed_u64(part + (size_t)(2 * c4) * H + h0, tg | __float_as_uint(Y[qs][s4][0]));
                        st_relaxed_u64(part + (size_t)(2 * c4) * H + h0 + 8, tg | __float_as_uint(Y[qs][s4][2]));
                    }
                    if (2 * c4 + 1 < T) {
                        st_relaxed_u64(part + (size_t)(2 * c4 + 1) * H + h0, tg | __float_as_uint(Y[qs][s4][1]));
                        st_relaxed_u64(part + (size_t)(2 * c4 + 1) * H + h0 + 8, tg | __float_as_uint(Y[qs][s4][3]));
                    }
                }
            }
        }
    }
    __syncthreads();
    // every CTA arrives once per launch, on every path, so the counts stay in lockstep
    if (tid == 0) arrive_relaxed(p.epoch + G);
    if (tracing && tid == 0) stamp(trace, 21);

    // ---- 5. output columns [16c, 16c + 16): every CTA's partial, summed in CTA order -------
    if ((int)blockIdx.x < H / 16) {
        const unsigned long long t_poll = globaltimer_ns();
        if (tid == 0) {
            // all but the last few CTAs arrived (the tags decide what is there)
            // (tests: extra_arrivals = 1 waits for a whole launch more, which never comes)
            const unsigned long long target =
                S.target + (unsigned long long)p.extra_arrivals * (unsigned long long)G - kDecArriveSlack;
            while ((long long)(ld_relaxed_u64(p.epoch + G) - target) < 0) {
                if (globaltimer_ns() - t_poll > p.exchange_timeout_ns) {
                    atomicOr(p.status, kDevBarrierTimeout);
                    S.abort = 1;
                    break;
                }
            }
            if (tracing) stamp(trace, 26);
        }
        __syncthreads();
        if (!S.abort) {
            // thread (slot, n) reads CTAs slot, slot + 16, ... of column 16c + n, all at
            // once, then again only the words without this launch's tag; the sums run in
            // CTA order, then over the 16 slots in order
            const int n = tid & 15, slot = tid >> 4;
            constexpr int PER = (kDecMaxCtas + kDecSlots - 1) / kDecSlots;
            float* ysum = red;   // [T][kDecSlots][16]
            const unsigned long long* col = p.part + 16 * blockIdx.x + n;
            const unsigned tag = S.tag;
            bool late = false;
            for (int t = 0; t < T; ++t) {
                unsigned long long v[PER];
                uint32_t pending = 0;
#pragma unroll
                for (int q = 0; q < PER; ++q) {
                    const int cta = slot + kDecSlots * q;
                    v[q] = cta < G ? ld_relaxed_u64(col + ((size_t)cta * T + t) * H) : ((unsigned long long)tag << 32);
                    if ((unsigned)(v[q] >> 32) != tag) pending |= 1u << q;
                }
                while (pending && !late) {
                    __nanosleep(64);
#pragma unroll
                    for (int q = 0; q < PER; ++q) {
                        if ((pending >> q) & 1u) {
                            v[q] = ld_relaxed_u64(col + ((size_t)(slot + kDecSlots * q) * T + t) * H);
                            if ((unsigned)(v[q] >> 32) == tag) pending &= ~(1u << q);
                        }
                    }
                    late = globaltimer_ns() - t_poll > p.exchange_timeout_ns;
                }
                float acc = 0.0f;
#pragma unroll
                for (int q = 0; q < PER; ++q) acc += __uint_as_float((uint32_t)v[q]);
                ysum[(t * kDecSlots + slot) * 16 + n] = acc;
            }
            if (late) {
                atomicOr(p.status, kDevBarrierTimeout);
                S.abort = 1;
            }
            if (tracing && tid == 0) stamp(trace, 23);
            __syncthreads();
            if (tid < 16 * T && !S.abort) {
                const int t = tid >> 4;
                float yv = 0.0f;
#pragma unroll
                for (int sl = 0; sl < kDecSlots; ++sl) yv += ysum[(t * kDecSlots + sl) * 16 + n];
                reinterpret_cast<__nv_bfloat16*>(p.y)[(size_t)t * H + 16 * blockIdx.x + n] = __float2bfloat16_rn(yv);
            }
        }
    }
    if (tracing && tid == 0) stamp(trace, 5);

    // ---- 6. never leave with copies in flight ------------------------------------------
    if (S.abort && tid == 0) {
        for (int u = 0; u < nu; ++u) {
            mbar_wait0(bar_gu(u), p.timeout_ns);
            if (S.dn_bytes[u] > 0) mbar_wait0(bar_dn(u), p.timeout_ns);
        }
    }
}

}  // namespace fe
