// A stack of decode layers, one token per persistent launch.
//
// "FireEcho Engine", sections "Benchmark Results" (row L6: the 48-layer
// forward captured as one CUDA graph; row L2: the next layer pinned in L2
// ahead of use) and "Speed Optimization History" (single-token decode path,
// multi-expert kernel, packed contiguous expert buffer).  Each layer is the
// layer of decode.cuh, split the same way along the intermediate dimension
// (units of 16 act columns of one routed expert, gate_up and the matching 16
// rows of W_dn per unit, a per-CTA partial y summed over the CTAs in a fixed
// order), but one CTA per SM runs every layer of the stack in turn, so that:
//
//   * every layer's router logits are inputs, so all layers are routed once
//     at the start (8 warps, each a share of the layers), and the weight
//     stream of a layer never waits for its routing;
//   * a CTA's units of all layers form one sequence streamed through a ring of
//     kStkSlots shared-memory slots: a slot is refilled (cp.async.bulk, one
//     mbarrier per copy) as soon as its unit is done, so the next layer's
//     weights arrive while the current layer finishes, and the stream does
//     not stop at layer boundaries;
//   * the unit split and the output slices a CTA sums rotate from layer to
//     layer (CTA c takes the share of c + 53 l mod G), so the CTAs that hold
//     one unit more than the others differ from layer to layer;
//   * sixteen compute warps run the units; a copy warp refills each ring slot
//     the moment its unit is done, an exchange warp stages the next layer's x
//     (fp16, double-buffered) and sums this CTA's output slices of finished
//     layers, and a sync warp makes the per-layer arrivals and clears each
//     partial buffer for reuse ahead of time, so none of those global-memory
//     round trips sits between the compute warps' units;
//   * the partials of the layers sit in six rotating buffers of tagged
//     64-bit words (launch, layer), with a count of summed slices per buffer
//     that a CTA checks before it reuses the buffer; with chained layers (layer l + 1
//     reads layer l's y) the exchange warp stages x_{l+1} once every slice of
//     y_l is written.
//
// A stack call at a few tokens whose routing is sparse runs one launch per token
// (layer rows T apart; launch 0 also writes every token's routing and grouping).
//
// Every wait is bounded by %globaltimer; the grid is one CTA per SM, all
// resident at once (checked on the host from the kernel's occupancy).
#pragma once

#include "bulk.cuh"
#include "common.cuh"
#include "decode.cuh"
#include "mma.cuh"
#include "warp_route.cuh"

namespace fe {

constexpr int kStkWarps = 16;         // compute warps
constexpr int kStkCompute = 32 * kStkWarps;
constexpr int kStkThreads = kStkCompute + 96;   // + the copy, exchange and sync warps
constexpr int kStkSlots = 3;          // unit ring
constexpr int kStkMaxLayers = 64;
constexpr int kStkMaxK = 16;
constexpr int kStkBufs = 6;           // partial-output buffers, by layer mod 6
constexpr int kStkRotate = 53;        // rotation of the unit split and the output slices per layer
constexpr int kStkRouteWarps = 8;     // warps routing the layers at the start
constexpr int kStkCand = 256;         // candidate keys per routing warp (k * E/32 at most)
constexpr int kStkMaxTokens = 4;      // tokens of a stack call run as one launch each, at most
constexpr int kStkRedFloats = 4096;   // routing candidates (8 x 256 keys); later the gate_up partials
constexpr int kStkPartFloats = 512;   // gate_up partials: 16 warps x 32
constexpr int kStkLandRow = 128;      // bytes of one CTA's share of one output slice (16 tagged words)
constexpr int kStkHQ = kDecMaxH / 64 / kStkWarps;   // output quads per warp

struct StackLayer {
    const uint8_t* gu_blocks;   // the layer's gate_up units (decode.cuh)
    const uint8_t* dn_rows;     // the layer's W_dn row groups (pack.cuh)
    int32_t* idx;               // the layer's routing outputs (its handle's workspace)
    float* w;
    int32_t* counts;
    int32_t* offsets;
    int32_t* sorted_pair;
    int32_t* pair_row;
};

struct StackParams {
    const StackLayer* layers;   // [L], device memory
    int L, E, H, I, k;
    const uint16_t* x;          // layer l reads the row x + l*ldx (bf16)
    const float* logits;        // layer l: the row logits + l*ldl
    uint16_t* y;                // layer l writes the row y + l*ldy
    size_t ldx, ldl, ldy;       // elements from one layer's row to the next (H, E, H for one token)
    int T, t;                   // this launch computes token t of the layers' T tokens (x, logits and y
                                //   point at token t's rows; launch t = 0 also writes every token's routing)
    int chained;                // y + l*ldy == x + (l+1)*ldx
    unsigned long long* part;   // [kStkBufs][grid][H]: (tag << 32) | fp32 bits; within each 16-column
                                //   tile, word 2g holds column g and word 2g + 1 column g + 8
    unsigned long long* ctr;    // [grid + 2 kStkBufs]: launches of CTA c; then per partial buffer b
                                //   (the layers l with l % kStkBufs = b) the CTAs' arrivals, and
                                //   then per buffer the output slices summed
    uint32_t* status;
    unsigned long long timeout_ns;
    unsigned long long* trace;   // optional [grid][16]: clock64 cycles thread 0 spent per phase, summed
};

// Phases of the optional trace (slots of each CTA's row).
enum StackPhase {
    kPhStage = 0,     // waiting for x and staging it
    kPhWaitGu = 1,    // waiting for a unit's gate_up bytes
    kPhGateUp = 2,    // gate_up mma
    kPhAct = 3,       // the warps' partials summed, SwiGLU, the down B column
    kPhWaitDn = 4,    // waiting for a unit's down bytes
    kPhDown = 5,      // down mma
    kPhSlot = 6,      // end-of-unit barrier and the next copy
    kPhGuard = 7,     // waiting until the partial buffer of the layer is free
    kPhPartial = 8,   // partial stores and the arrival
    kPhUnits = 9,     // units processed
    kPhTotal = 10,    // the whole layer loop
    // the exchange warp (lane 0)
    kPhHPoll = 11,    // cycles in arrival and slice-count polls
    kPhHPolls = 12,   // polls
    kPhHSum = 13,     // cycles summing output slices
    kPhHLand = 14,    // cycles landing the slices' words (cp.async)
    kPhHAdd = 15      // cycles adding them up
};

struct StackShared {
    int dex[kStkMaxLayers][kStkMaxK];   // routed experts of each layer, ascending
    float dw[kStkMaxLayers][kStkMaxK];  // slot weight of each
    int rsel_e[kStkRouteWarps][kStkMaxK];
    float rsel_w[kStkRouteWarps][kStkMaxK];
    const uint8_t* gu[kStkMaxLayers];
    const uint8_t* dn[kStkMaxLayers];
    uint32_t bfrag[8];                  // current unit's down B column (token 0), f16x2
    int bshift;
    int xshift[2];                      // shift of the x row staged in xs buffer b
    volatile int xs_layer[2];           // layer whose x is staged in xs buffer b (exchange -> compute)
    volatile int layer_done;            // last layer whose units and partial are done (compute -> exchange)
    volatile int guard_ok;              // last layer whose partial buffer is free (sync -> compute)
    volatile int abort;
    unsigned long long epoch;
};

struct StackSmem {
    uint32_t mbar, shared, red, land, xs, xr, total;
};

__host__ __device__ inline StackSmem stack_smem_layout(int H)
{
    StackSmem L;
    L.mbar = (uint32_t)kStkSlots * dec_unit_bytes(H);
    L.shared = L.mbar + 8 * (3 * kStkSlots + 2);
    L.red = align16(L.shared + (uint32_t)sizeof(StackShared));
    static_assert(kStkRedFloats * 4 >= kStkRouteWarps * kStkCand * 8, "routing candidates space");
    static_assert(2 * kStkMaxTokens * kStkMaxK * 4 <= kStkCand * 8, "grouping of a few tokens in the candidates' space");
    // after routing, the candidates' space holds the gate_up partials and, behind them,
    // the landing rows of an output slice (one 128-byte row per CTA, written by cp.async)
    L.land = L.red + 4u * kStkPartFloats;
    const uint32_t after = L.land + (uint32_t)kDecMaxCtas * kStkLandRow;
    L.xs = align16(after > L.red + 4u * kStkRedFloats ? after : L.red + 4u * kStkRedFloats);
    L.xr = align16(L.xs + 4u * 3 * brow_words(H));   // two x rows (double buffer) + the zero row
    L.total = align16(L.xr + 2u * 2 * H);
    return L;
}

__host__ __device__ inline unsigned stack_tag(unsigned long long epoch, int L, int l)
{
    return (unsigned)((epoch * (unsigned long long)L + (unsigned long long)l) % 0xffffffffull) + 1u;
}

// A per-buffer count (arrivals: `per_layer` = grid; summed slices: H / 16) once
// every event of layer l, and so of every earlier layer of buffer l % kStkBufs in
// this launch and all earlier ones, has been counted.  One count per buffer: an
// event of a later layer of another buffer can come before the last one of
// layer l, and a single running count would pass its target too early.
__host__ __device__ inline unsigned long long stack_count_through(unsigned long long epoch, int L, int l,
                                                                   int per_layer)
{
    const int b = l % kStkBufs;
    const unsigned long long nb = (unsigned long long)((L - b + kStkBufs - 1) / kStkBufs);   // layers of buffer b
    return (epoch * nb + (unsigned long long)(l / kStkBufs) + 1ull) * (unsigned long long)per_layer;
}

// This CTA's share of layer l's U units: [first, first + n).
FE_DEV void stack_units(int c, int l, int U, int G, int& first, int& n)
{
    const int v = (c + l * kStkRotate) % G;
    first = dec_unit_first(v, U, G);
    n = dec_unit_first(v + 1, U, G) - first;
}

__global__ void __launch_bounds__(kStkThreads, 1) stack_decode_kernel(StackParams p)
{
    extern __shared__ __align__(128) uint8_t ssm[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, c4 = lane & 3;
    const int L = p.L, E = p.E, H = p.H, I = p.I, k = p.k;
    const int G = gridDim.x, c = blockIdx.x;
    const StackSmem SL = stack_smem_layout(H);
    const uint32_t gu_unit = 2u * block_bytes(H), slot_bytes = dec_unit_bytes(H);
    const int xrw = brow_words(H), upe = I / 16, U = k * upe, nq = H / 64;
    uint8_t* slots = ssm;
    StackShared& S = *reinterpret_cast<StackShared*>(ssm + SL.shared);
    float* red = reinterpret_cast<float*>(ssm + SL.red);
    uint32_t* xs = reinterpret_cast<uint32_t*>(ssm + SL.xs);   // rows: x buffer 0, x buffer 1, zeros
    uint16_t* xr = reinterpret_cast<uint16_t*>(ssm + SL.xr);
    const uint32_t mbar0 = smem_addr(ssm + SL.mbar);
    auto bar_gu = [&](int s) { return mbar0 + 8u * (uint32_t)s; };
    auto bar_dn = [&](int s) { return mbar0 + 8u * (uint32_t)(kStkSlots + s); };
    auto bar_x = [&](int b) { return mbar0 + 8u * (uint32_t)(2 * kStkSlots + b); };
    // slot s is free again once every compute warp has arrived (one arrival per warp per unit)
    auto bar_empty = [&](int s) { return mbar0 + 8u * (uint32_t)(2 * kStkSlots + 2 + s); };
    const bool copier = warp == kStkWarps, exchanger = warp == kStkWarps + 1, syncer = warp == kStkWarps + 2;
    // diagnostics: compute thread 0's cycles per phase
    unsigned long long ph_acc[11] = {};
    long long ph_t = 0;
    const bool tracing = p.trace != nullptr && tid == 0;
    auto ph_start = [&]() { if (tracing) ph_t = clock64(); };
    auto ph_end = [&](int ph) { if (tracing) { const long long t = clock64(); ph_acc[ph] += (unsigned long long)(t - ph_t); ph_t = t; } };
    // the compute warps' own barrier (the copy and exchange warps never join it)
    auto cbar = []() { asm volatile("bar.sync 1, %0;" ::"n"(kStkCompute) : "memory"); };

    if (tid == 0) {
        for (int b = 0; b < 2 * kStkSlots + 2; ++b) mbar_init(mbar0 + 8u * b, 1);
        for (int s = 0; s < kStkSlots; ++s) mbar_init(bar_empty(s), kStkWarps);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        S.abort = 0;
        S.layer_done = -1;
        S.guard_ok = kStkBufs - 1;   // the first kStkBufs layers' buffers are free
        S.xs_layer[0] = -1;
        S.xs_layer[1] = -1;
    }
    for (int i = tid; i < xrw; i += kStkThreads) xs[2 * xrw + i] = 0u;   // the zero B row
    if (tid < 8) S.bfrag[tid] = 0u;
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (tid == 0) {
        const unsigned long long ep = *reinterpret_cast<volatile unsigned long long*>(p.ctr + c);
        S.epoch = ep;
        p.ctr[c] = ep + 1ull;   // every CTA runs every launch: the counts move in lockstep
    }
    // the layers' weight pointers
    for (int l = tid; l < L; l += kStkThreads) {
        S.gu[l] = p.layers[l].gu_blocks;
        S.dn[l] = p.layers[l].dn_rows;
    }
    // ---- route every layer: warp w < 8 takes layers w, w + 8, ... ----------------------
    if (warp < kStkRouteWarps) {
        unsigned long long* cand = reinterpret_cast<unsigned long long*>(red) + warp * kStkCand;
        int* se = S.rsel_e[warp];
        float* sw = S.rsel_w[warp];
        for (int l = warp; l < L; l += kStkRouteWarps) {
            const bool nan = warp_route(p.logits + (size_t)l * p.ldl, E, k, lane, cand, kStkCand, se, sw);
            if (nan && lane == 0) atomicOr(p.status, kDevNanLogit);
            warp_softmax(sw, k, lane);
            int pos = 0;
            if (lane < k) {
                for (int q = 0; q < k; ++q) pos += se[q] < se[lane];
                S.dex[l][pos] = se[lane];
                S.dw[l][pos] = sw[lane];
            }
            // the layer's routing outputs, from one CTA per layer: at one token, this one;
            // with T tokens (one launch each), launch 0 routes them all (below)
            if (c == l % G && p.T == 1) {
                const StackLayer& ly = p.layers[l];
                if (lane < k) {
                    ly.idx[lane] = se[lane];
                    ly.w[lane] = sw[lane];
                    ly.sorted_pair[pos] = lane;
                    ly.pair_row[lane] = pos;
                }
                for (int e = lane; e <= E; e += 32) {
                    int below = 0, eq = 0;
                    for (int q = 0; q < k; ++q) {
                        below += se[q] < e;
                        eq += se[q] == e;
                    }
                    ly.offsets[e] = below;
                    if (e < E) ly.counts[e] = eq;
                }
            }
            if (c == l % G && p.T > 1 && p.t == 0) {
                // every token of the layer routed (idx, w in slot order), then the pairs p =
                // t*k + j grouped: the rank of a pair by (expert, pair id), and the offsets by
                // binary search in the sorted experts, in the candidates' space (free again)
                const StackLayer& ly = p.layers[l];
                const int P = p.T * k;
                for (int tt = 0; tt < p.T; ++tt) {
                    warp_route(p.logits + (size_t)l * p.ldl + (size_t)tt * E, E, k, lane, cand, kStkCand, se, sw);
                    warp_softmax(sw, k, lane);
                    if (lane < k) {
                        ly.idx[tt * k + lane] = se[lane];
                        ly.w[tt * k + lane] = sw[lane];
                    }
                    __syncwarp();
                }
                int* sidx = reinterpret_cast<int*>(cand);
                int* ssort = sidx + kStkMaxTokens * kStkMaxK;
                for (int q = lane; q < P; q += 32) sidx[q] = ly.idx[q];
                __syncwarp();
                for (int q = lane; q < P; q += 32) {
                    const int eq = sidx[q];
                    int rank = 0;
                    for (int r = 0; r < P; ++r) {
                        const int er = sidx[r];
                        rank += er < eq || (er == eq && r < q);
                    }
                    ssort[rank] = eq;
                    ly.sorted_pair[rank] = q;
                    ly.pair_row[q] = rank;
                }
                __syncwarp();
                for (int e = lane; e <= E; e += 32) {
                    int lo = 0, hi = P;   // first sorted position with expert >= e
                    while (lo < hi) {
                        const int m = (lo + hi) >> 1;
                        if (ssort[m] < e) lo = m + 1; else hi = m;
                    }
                    int lo2 = lo, hi2 = P;   // ... and with expert > e
                    while (lo2 < hi2) {
                        const int m = (lo2 + hi2) >> 1;
                        if (ssort[m] <= e) lo2 = m + 1; else hi2 = m;
                    }
                    ly.offsets[e] = lo;
                    if (e < E) ly.counts[e] = lo2 - lo;
                }
                __syncwarp();
            }
            __syncwarp();
        }
    }
    __syncthreads();
    const unsigned long long epoch = S.epoch;

    if (copier) {
        // ==== the copy warp: unit q of this CTA's sequence goes into slot q % 3 as soon
        // as every compute warp has arrived on the slot's empty barrier for unit q - 3.
        // Lane 0 alone; nothing else in the loop, so that a freed slot is refilled at once.
        if (lane != 0) return;
        int total = 0;
        for (int l = 0; l < L; ++l) {
            int f, n;
            stack_units(c, l, U, G, f, n);
            total += n;
        }
        int pl = 0, pi = 0, pf = 0, pc = 0;   // next unit: layer, index, layer's first unit and count
        stack_units(c, 0, U, G, pf, pc);
        int issued = 0;
        for (; issued < total; ++issued) {
            if (issued >= kStkSlots) {
                // use (issued - 3) / 3 of the slot: phases complete in order, and the next
                // one cannot complete before this copy is issued
                const uint32_t ph = (uint32_t)((issued - kStkSlots) / kStkSlots) & 1u;
                if (!S.abort && !mbar_wait(bar_empty(issued % kStkSlots), ph, p.timeout_ns)) {
                    atomicOr(p.status, kDevBarrierTimeout);
                    S.abort = 1;
                }
                if (S.abort) break;
            }
            while (pi >= pc) {
                ++pl;
                pi = 0;
                stack_units(c, pl, U, G, pf, pc);
            }
            const int s = issued % kStkSlots;
            const int u = pf + pi, d = u / upe, j = u - d * upe, e = S.dex[pl][d];
            const uint32_t base = smem_addr(slots) + (uint32_t)s * slot_bytes;
            mbar_expect_tx(bar_gu(s), gu_unit);
            mbar_expect_tx(bar_dn(s), 10u * H);
            bulk_g2s(base, S.gu[pl] + ((size_t)e * upe + j) * gu_unit, gu_unit, bar_gu(s));
            bulk_g2s(base + gu_unit,
                     S.dn[pl] + ((size_t)e * (I / 32) + j / 2) * 18ull * H + ((j & 1) ? 8ull * H : 0ull), 10u * H,
                     bar_dn(s));
            ++pi;
        }
        // never leave with copies in flight: wait (bounded) for the last copy issued
        // into each slot (phases complete in order)
        for (int q = issued > kStkSlots ? issued - kStkSlots : 0; q < issued; ++q) {
            const uint32_t ph = (uint32_t)(q / kStkSlots) & 1u;
            mbar_wait(bar_gu(q % kStkSlots), ph, p.timeout_ns);
            mbar_wait(bar_dn(q % kStkSlots), ph, p.timeout_ns);
        }
    } else if (syncer) {
        // ==== the sync warp (lane 0): the global-memory handshakes whose round trips would
        // otherwise sit on the compute warps' path.  It makes this CTA's arrival for every
        // layer whose partial is stored (a release, so the partial is visible first) and
        // polls the summed-slice counts, so that each partial buffer is known free before
        // the compute warps reach the layer that reuses it.
        if (lane != 0) return;
        int al = 0;          // next layer to arrive for
        int gl = kStkBufs;   // next layer whose buffer to clear
        const unsigned long long t_start = globaltimer_ns();
        bool late = false;
        while ((al < L || gl < L) && !late) {
            bool progress = false;
            if (al < L && S.layer_done >= al) {
                __threadfence_block();
                arrive_release(p.ctr + G + al % kStkBufs);
                ++al;
                progress = true;
            }
            if (gl < L && !S.abort) {
                const unsigned long long target = stack_count_through(epoch, L, gl - kStkBufs, H / 16);
                if ((long long)(ld_acquire_u64(p.ctr + G + kStkBufs + gl % kStkBufs) - target) >= 0) {
                    S.guard_ok = gl;
                    ++gl;
                    progress = true;
                }
            }
            if (S.abort) gl = L;   // the compute warps no longer wait on it
            if (!progress) late = globaltimer_ns() - t_start > p.timeout_ns * 4;
        }
        if (late) {
            atomicOr(p.status, kDevBarrierTimeout);
            S.abort = 1;
        }
        // every layer's arrival is made on every path (after an abort the compute warps skip
        // their work and still publish each layer), so that later launches' counts stay in
        // lockstep with the launch count
        for (; al < L; ++al) arrive_release(p.ctr + G + al % kStkBufs);
    } else if (exchanger) {
        // ==== the exchange warp ================================================================
        // Event loop over two jobs, each taken as soon as it can proceed: stage the next
        // layer's x when its buffer and its bytes are there, sum this CTA's output slice of
        // the oldest finished layer when all its partials are in.
        int xl = 0;                           // next layer to stage
        int rl = 0;                           // next layer to sum
        unsigned long long* land = reinterpret_cast<unsigned long long*>(ssm + SL.land);
        int xin = p.chained ? 1 : (L < 2 ? L : 2);   // x rows copied into xr so far (layers 0 .. xin-1)
        if (lane == 0) {
            for (int l = 0; l < xin; ++l) {
                mbar_expect_tx(bar_x(l), 2u * H);
                bulk_g2s(smem_addr(xr + (size_t)l * H), p.x + (size_t)l * p.ldx, 2u * H, bar_x(l));
            }
        }
        const unsigned long long t_start = globaltimer_ns();
        bool late = false;
        // every decision of the loop is taken by lane 0 and broadcast, so that the
        // lanes never disagree on a branch (the flags change under their feet)
        auto uniform = [&](bool v) { return __shfl_sync(0xffffffffu, (int)v, 0) != 0; };
        const bool htrace = p.trace != nullptr && lane == 0;
        unsigned long long h_poll = 0, h_polls = 0, h_sum = 0, h_land = 0, h_add = 0;
        while ((xl < L || rl < L) && !late) {
            bool progress = false;
            const int ldone = __shfl_sync(0xffffffffu, S.layer_done, 0);
            // -- x of layer xl into xs buffer xl & 1, once the compute warps are done with
            //    layer xl - 2 (which used it) and x_xl is there
            if (xl < L && ldone >= xl - 2) {
                bool ready = false;
                if (lane == 0) {
                    if (p.chained && xl > 0) {
                        const unsigned long long target = stack_count_through(epoch, L, xl - 1, H / 16);
                        ready = (long long)(ld_acquire_u64(p.ctr + G + kStkBufs + (xl - 1) % kStkBufs) - target) >= 0;
                    } else {
                        ready = mbar_test(bar_x(xl & 1), (uint32_t)(xl >> 1) & 1u);
                    }
                }
                if (uniform(ready)) {
                    const bool global_src = p.chained && xl > 0;
                    const uint32_t* src = global_src ? reinterpret_cast<const uint32_t*>(p.x + (size_t)xl * p.ldx)
                                                     : reinterpret_cast<const uint32_t*>(xr + (size_t)(xl & 1) * H);
                    float m = 0.0f;
                    for (int r = lane; r < H / 2; r += 32) {
                        const uint32_t two = global_src ? __ldcg(src + r) : src[r];
                        m = fmaxf(m, fmaxf(fabsf(bf16_bits_to_f32((uint16_t)(two & 0xffff))),
                                           fabsf(bf16_bits_to_f32((uint16_t)(two >> 16)))));
                    }
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                    const int sh = fp16_shift(m);
                    const float scl = pow2f(-sh);
                    uint32_t* dst = xs + (size_t)(xl & 1) * xrw;
                    for (int r = lane; r < H / 2; r += 32) {
                        const uint32_t two = global_src ? __ldcg(src + r) : src[r];
                        dst[bfrag_word(r)] = f32x2_to_f16x2_rn(bf16_bits_to_f32((uint16_t)(two & 0xffff)) * scl,
                                                               bf16_bits_to_f32((uint16_t)(two >> 16)) * scl);
                    }
                    __syncwarp();
                    if (lane == 0) {
                        S.xshift[xl & 1] = sh;
                        __threadfence_block();
                        S.xs_layer[xl & 1] = xl;
                        // the row buffer just read takes layer xl + 2's x
                        if (!p.chained && xl + 2 < L) {
                            mbar_expect_tx(bar_x(xl & 1), 2u * H);
                            bulk_g2s(smem_addr(xr + (size_t)(xl & 1) * H), p.x + (size_t)(xl + 2) * p.ldx, 2u * H,
                                     bar_x(xl & 1));
                            ++xin;
                        }
                    }
                    ++xl;
                    progress = true;
                }
            }
            // -- this CTA's output slice of layer rl, once every CTA has arrived
            if (rl < L && ldone >= rl) {
                const int sl = (c + rl * kStkRotate) % G;
                if (sl >= H / 16) {
                    ++rl;   // no slice of this layer here
                    progress = true;
                } else {
                    const unsigned long long target = stack_count_through(epoch, L, rl, G);
                    bool all_in = false;
                    if (lane == 0) {
                        const long long tp = htrace ? clock64() : 0;
                        all_in = (long long)(ld_acquire_u64(p.ctr + G + rl % kStkBufs) - target) >= 0;
                        if (htrace) { h_poll += (unsigned long long)(clock64() - tp); ++h_polls; }
                    }
                    if (uniform(all_in)) {
                        const long long ts = htrace ? clock64() : 0;
                        // lane (grp, cp) adds columns 16 sl + cp, + 8 over CTAs grp, grp + 4,
                        // ... in order, and the four groups are added in order.  Its 16-byte
                        // words first land in shared memory (cp.async: every load of the slice
                        // in flight at once, no registers held), one round trip in all
                        const int cp = lane & 7, grp = lane >> 3;
                        const unsigned tag = stack_tag(epoch, L, rl);
                        const unsigned long long* col = p.part + (size_t)(rl % kStkBufs) * G * H + 16 * sl;
                        __syncwarp();   // lane 0's acquire above, for every lane
                        for (int cta = grp; cta < G; cta += 4)
                            cp_async16_cg(smem_addr(land + (size_t)cta * (kStkLandRow / 8) + 2 * cp),
                                          col + (size_t)cta * H + 2 * cp);
                        cp_async_wait_all();
                        const long long tl = htrace ? clock64() : 0;
                        if (htrace) h_land += (unsigned long long)(tl - ts);
                        float a0 = 0.0f, a1 = 0.0f;
                        unsigned bad = 0u;   // a landed word of another launch or layer
#pragma unroll 4
                        for (int cta = grp; cta < G; cta += 4) {
                            const ulonglong2 v =
                                *reinterpret_cast<const ulonglong2*>(land + (size_t)cta * (kStkLandRow / 8) + 2 * cp);
                            bad |= ((unsigned)(v.x >> 32) ^ tag) | ((unsigned)(v.y >> 32) ^ tag);
                            a0 += __uint_as_float((uint32_t)v.x);
                            a1 += __uint_as_float((uint32_t)v.y);
                        }
                        if (__any_sync(0xffffffffu, bad != 0u)) {
                            // a word that was not there yet (the arrivals are released after the
                            // stores, so this is not expected): the sum again, from global
                            // memory, each word read until its tag is there (bounded)
                            a0 = 0.0f;
                            a1 = 0.0f;
                            for (int cta = grp; cta < G && !late; cta += 4) {
                                ulonglong2 v = ld_relaxed_u64x2(col + (size_t)cta * H + 2 * cp);
                                while (((unsigned)(v.x >> 32) != tag || (unsigned)(v.y >> 32) != tag) && !late) {
                                    __nanosleep(32);
                                    v = ld_relaxed_u64x2(col + (size_t)cta * H + 2 * cp);
                                    late = globaltimer_ns() - t_start > p.timeout_ns;
                                }
                                a0 += __uint_as_float((uint32_t)v.x);
                                a1 += __uint_as_float((uint32_t)v.y);
                            }
                        }
                        late = __any_sync(0xffffffffu, late);
                        if (htrace) h_add += (unsigned long long)(clock64() - tl);
                        const float b0 = __shfl_sync(0xffffffffu, a0, cp), b1 = __shfl_sync(0xffffffffu, a1, cp);
                        const float c0v = __shfl_sync(0xffffffffu, a0, cp + 8), c1v = __shfl_sync(0xffffffffu, a1, cp + 8);
                        const float d0 = __shfl_sync(0xffffffffu, a0, cp + 16), d1 = __shfl_sync(0xffffffffu, a1, cp + 16);
                        const float e0 = __shfl_sync(0xffffffffu, a0, cp + 24), e1 = __shfl_sync(0xffffffffu, a1, cp + 24);
                        if (grp == 0 && !late) {   // words 2cp, 2cp + 1 of a tile: columns cp, cp + 8
                            const uint32_t two = bf16x2_rn(((b0 + c0v) + d0) + e0, ((b1 + c1v) + d1) + e1);
                            uint16_t* yr = p.y + (size_t)rl * p.ldy + 16 * sl;
                            yr[cp] = (uint16_t)(two & 0xffffu);
                            yr[cp + 8] = (uint16_t)(two >> 16);
                        }
                        if (p.chained) __threadfence();   // the slice is visible before it is counted
                        __syncwarp();
                        // counted on every path (release: the partials have been read), in every
                        // launch: the counts stay in lockstep with the launch count
                        if (lane == 0) arrive_release(p.ctr + G + kStkBufs + rl % kStkBufs);
                        if (htrace) h_sum += (unsigned long long)(clock64() - ts);
                        ++rl;
                        progress = true;
                    }
                }
            }
            if (!progress) {
                __nanosleep(64);
                late = uniform(globaltimer_ns() - t_start > p.timeout_ns * 4);
            }
            __syncwarp();
        }
        if (htrace) {
            unsigned long long* row = p.trace + (size_t)c * 16;
            row[kPhHPoll] = h_poll;
            row[kPhHPolls] = h_polls;
            row[kPhHSum] = h_sum;
            row[kPhHLand] = h_land;
            row[kPhHAdd] = h_add;
        }
        if (late && lane == 0) {
            atomicOr(p.status, kDevBarrierTimeout);
            S.abort = 1;
            // the slices not summed are still counted, so that the counts of later
            // launches stay in lockstep with the launch count
            for (; rl < L; ++rl)
                if ((c + rl * kStkRotate) % G < H / 16) arrive_release(p.ctr + G + kStkBufs + rl % kStkBufs);
        }
        // never leave with a copy in flight: wait (bounded) for the last x rows
        if (lane == 0)
            for (int l = xin > 2 ? xin - 2 : 0; l < xin; ++l)
                mbar_wait(bar_x(l & 1), (uint32_t)(l >> 1) & 1u, p.timeout_ns);
    } else {
        // ==== the compute warps ================================================================
        int n = 0;   // unit sequence index
        const long long t_loop = clock64();
        for (int l = 0; l < L; ++l) {
            ph_start();
            // x of this layer, staged by the exchange warp
            if (tid == 0) {
                const unsigned long long t0 = globaltimer_ns();
                while (S.xs_layer[l & 1] != l && !S.abort) {
                    if (globaltimer_ns() - t0 > p.timeout_ns) {
                        atomicOr(p.status, kDevLoadTimeout);
                        S.abort = 1;
                    }
                }
            }
            cbar();
            const float xm = pow2f(S.xshift[l & 1]);
            const uint32_t* xrow = xs + (size_t)(l & 1) * xrw;
            ph_end(kPhStage);

            float Y[kStkHQ][4][4];
#pragma unroll
            for (int a = 0; a < kStkHQ; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b)
#pragma unroll
                    for (int d2 = 0; d2 < 4; ++d2) Y[a][b][d2] = 0.0f;
            int u0, nu;
            stack_units(c, l, U, G, u0, nu);
            for (int i = 0; i < nu; ++i, ++n) {
                const int s = n % kStkSlots;
                const uint32_t ph = (uint32_t)(n / kStkSlots) & 1u;
                const int u = u0 + i, d = u / upe, j = u - d * upe;
                if (!S.abort && !mbar_wait(bar_gu(s), ph, p.timeout_ns)) {
                    atomicOr(p.status, kDevLoadTimeout);
                    S.abort = 1;
                }
                ph_end(kPhWaitGu);
                const uint8_t* blk0 = slots + (size_t)s * slot_bytes;
                const uint8_t* blk1 = blk0 + block_bytes(H);
                // gate_up: warp w takes the 64-k quads w, w + W, ...
                float t0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, t1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                const uint32_t* brow = g == 0 ? xrow : xs + 2 * xrw;
#pragma unroll 1
                for (int q = warp; q < nq; q += kStkWarps) {
                    uint32_t b[8];
                    load_bfrag(brow, q, lane, b);
                    quad_mma2_b(blk0, blk1, H, b, q, lane, t0, t1);
                }
                ph_end(kPhGateUp);
                if (c4 == 0) {   // token column 0: rows g, g + 8 of gate (t0) and up (t1)
                    float* rw = red + warp * 32;
                    rw[g] = t0[0];
                    rw[g + 8] = t0[2];
                    rw[16 + g] = t1[0];
                    rw[24 + g] = t1[2];
                }
                cbar();
                if (warp == 0) {
                    const int half = lane >> 4, cc = lane & 15;
                    float sacc = 0.0f;
#pragma unroll
                    for (int w2 = 0; w2 < kStkWarps; ++w2) sacc += red[w2 * 32 + half * 16 + cc];
                    const float other = __shfl_xor_sync(0xffffffffu, sacc, 16);
                    const float v = half == 0 ? silu_mul_fast(sacc * xm, other * xm) * S.dw[l][d] : 0.0f;
                    // the row max: non-negative floats order as their bits, so one warp reduction
                    // (the other half-warp holds zeros)
                    const float mx = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(v))));
                    const int sh = fp16_shift(mx);
                    const float sc = pow2f(-sh);
                    const float vn = __shfl_down_sync(0xffffffffu, v, 1);
                    if (half == 0 && (cc & 1) == 0) S.bfrag[cc >> 1] = f32x2_to_f16x2_rn(v * sc, vn * sc);
                    if (lane == 0) S.bshift = sh;
                }
                cbar();
                ph_end(kPhAct);
                if (!S.abort && !mbar_wait(bar_dn(s), ph, p.timeout_ns)) {
                    atomicOr(p.status, kDevLoadTimeout);
                    S.abort = 1;
                }
                ph_end(kPhWaitDn);
                if (!S.abort) {
                    const uint32_t b0 = g == 0 ? S.bfrag[c4] : 0u, b1 = g == 0 ? S.bfrag[c4 + 4] : 0u;
                    const float m0 = pow2f(S.bshift);
                    const uint8_t* codes = blk0 + gu_unit + ((j & 1) ? 2u * H : 0u);
                    const uint8_t* scl = blk0 + gu_unit + ((j & 1) ? 0u : 8u * H);
#pragma unroll
                    for (int qs = 0; qs < kStkHQ; ++qs) {
                        const int q = warp + kStkWarps * qs;
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
                                Y[qs][s4][0] = fmaf(dd[0], __uint_as_float(sw << 16) * m0, Y[qs][s4][0]);
                                Y[qs][s4][2] = fmaf(dd[2], __uint_as_float(sw & 0xffff0000u) * m0, Y[qs][s4][2]);
                            }
                        }
                    }
                }
                ph_end(kPhDown);
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_empty(s));   // this warp is done with the slot
                ph_end(kPhSlot);
                if (tracing) ph_acc[kPhUnits] += 1;
            }
            // this CTA's partial of layer l, tagged, then one arrival.  The buffer of layer
            // l held layer l - kStkBufs, whose slices other CTAs may still be summing (a CTA
            // can run ahead of them): wait until every slice of that layer has been summed
            // (the sync warp clears each buffer ahead of use)
            if (l >= kStkBufs) {
                if (tid == 0) {
                    const unsigned long long t0 = globaltimer_ns();
                    while (S.guard_ok < l && !S.abort) {
                        if (globaltimer_ns() - t0 > p.timeout_ns) {
                            atomicOr(p.status, kDevBarrierTimeout);
                            S.abort = 1;
                        }
                    }
                }
                cbar();
            }
            ph_end(kPhGuard);
            if (!S.abort) {
                unsigned long long* part = p.part + ((size_t)(l % kStkBufs) * G + c) * H;
                const unsigned long long tg = (unsigned long long)stack_tag(epoch, L, l) << 32;
                // the token's outputs sit in the lanes (g, 0): columns g and g + 8 of each
                // 16-column tile.  Lane (g, c4) takes tile 4q + c4 and stores its two columns
                // side by side (words 2g, 2g + 1 of the tile) in one 16-byte store
#pragma unroll
                for (int qs = 0; qs < kStkHQ; ++qs) {
                    const int q = warp + kStkWarps * qs;
                    float v0 = 0.0f, v1 = 0.0f;
#pragma unroll
                    for (int s4 = 0; s4 < 4; ++s4) {
                        const float a = __shfl_sync(0xffffffffu, Y[qs][s4][0], lane & ~3);
                        const float b = __shfl_sync(0xffffffffu, Y[qs][s4][2], lane & ~3);
                        if (c4 == s4) {
                            v0 = a;
                            v1 = b;
                        }
                    }
                    if (q < nq)
                        st_relaxed_u64x2(part + 16 * (4 * q + c4) + 2 * g, tg | __float_as_uint(v0),
                                         tg | __float_as_uint(v1));
                }
            }
            cbar();
            if (tid == 0) {
                // the sync warp makes the layer's arrival (a gpu-scope release) once it sees
                // the flag; the barrier and this fence order every compute thread's partial
                // stores before it
                __threadfence_block();
                S.layer_done = l;
            }
            ph_end(kPhPartial);
        }
        if (tracing) {
            ph_acc[kPhTotal] = (unsigned long long)(clock64() - t_loop);
            for (int q = 0; q < 11; ++q) p.trace[(size_t)c * 16 + q] = ph_acc[q];
        }
    }
}

}  // namespace fe
