// A stack of decode layers at one token in one persistent launch.
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
//   * with independent layers a CTA sums its output slice of layer l after its
//     first unit of layer l + 1 (the other CTAs' partials have arrived by
//     then), with the partials of the layers in three rotating buffers of
//     tagged 64-bit words (launch, layer) and a counter of summed slices that
//     a CTA checks before it reuses a buffer; with chained layers (layer l + 1
//     reads layer l's y) every CTA waits for all slices of y_l before it
//     stages its input.
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

constexpr int kStkThreads = 512;
constexpr int kStkWarps = kStkThreads / 32;
constexpr int kStkSlots = 3;          // unit ring
constexpr int kStkMaxLayers = 64;
constexpr int kStkMaxK = 16;
constexpr int kStkBufs = 3;           // partial-output buffers, by layer mod 3
constexpr int kStkRotate = 53;        // rotation of the unit split and the output slices per layer
constexpr int kStkRouteWarps = 8;     // warps routing the layers at the start
constexpr int kStkCand = 256;         // candidate keys per routing warp (k * E/32 at most)
constexpr int kStkRedFloats = 4096;   // candidates (8 x 256 keys), gate_up partials, final sums
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
    const uint16_t* x;          // layer l reads x + l*H (bf16)
    const float* logits;        // layer l: logits + l*E
    uint16_t* y;                // layer l writes y + l*H
    int chained;                // y + l*H == x + (l+1)*H
    unsigned long long* part;   // [kStkBufs][grid][H]: (tag << 32) | fp32 bits
    unsigned long long* ctr;    // [grid + 2]: launches of CTA c; arrivals; y slices written
    uint32_t* status;
    unsigned long long timeout_ns;
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
    int xshift;
    int abort;
    float wmax[kStkWarps];
    unsigned long long epoch;
};

struct StackSmem {
    uint32_t mbar, shared, red, xs, xr, total;
};

__host__ __device__ inline StackSmem stack_smem_layout(int H)
{
    StackSmem L;
    L.mbar = (uint32_t)kStkSlots * dec_unit_bytes(H);
    L.shared = L.mbar + 8 * (2 * kStkSlots + 2);
    L.red = align16(L.shared + (uint32_t)sizeof(StackShared));
    static_assert(kStkRedFloats * 4 >= kStkRouteWarps * kStkCand * 8, "routing candidates space");
    L.xs = L.red + 4u * kStkRedFloats;
    L.xr = align16(L.xs + 4u * 2 * brow_words(H));
    L.total = align16(L.xr + 2u * 2 * H);
    return L;
}

__host__ __device__ inline unsigned stack_tag(unsigned long long epoch, int L, int l)
{
    return (unsigned)((epoch * (unsigned long long)L + (unsigned long long)l) % 0xffffffffull) + 1u;
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
    uint32_t* xs = reinterpret_cast<uint32_t*>(ssm + SL.xs);
    uint16_t* xr = reinterpret_cast<uint16_t*>(ssm + SL.xr);
    const uint32_t mbar0 = smem_addr(ssm + SL.mbar);
    auto bar_gu = [&](int s) { return mbar0 + 8u * (uint32_t)s; };
    auto bar_dn = [&](int s) { return mbar0 + 8u * (uint32_t)(kStkSlots + s); };
    auto bar_x = [&](int b) { return mbar0 + 8u * (uint32_t)(2 * kStkSlots + b); };

    if (tid == 0) {
        for (int b = 0; b < 2 * kStkSlots + 2; ++b) mbar_init(mbar0 + 8u * b, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        S.abort = 0;
    }
    for (int i = tid; i < xrw; i += kStkThreads) xs[xrw + i] = 0u;   // row 1: the zero B row
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
            const bool nan = warp_route(p.logits + (size_t)l * E, E, k, lane, cand, kStkCand, se, sw);
            if (nan && lane == 0) atomicOr(p.status, kDevNanLogit);
            warp_softmax(sw, k, lane);
            int pos = 0;
            if (lane < k) {
                for (int q = 0; q < k; ++q) pos += se[q] < se[lane];
                S.dex[l][pos] = se[lane];
                S.dw[l][pos] = sw[lane];
            }
            // the layer's routing outputs, from one CTA per layer
            if (c == l % G) {
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
            __syncwarp();
        }
    }
    __syncthreads();
    const unsigned long long epoch = S.epoch;

    // ---- the producer (thread 0): units of the whole stack through the slot ring ------
    int pl = 0, pi = 0, pn_first = 0, pn_count = 0;   // next unit to issue: layer, index in the layer
    int issued = 0;                                    // units issued so far (sequence index)
    auto producer_next = [&]() -> bool {   // advance (pl, pi) to an existing unit; false at the end
        while (pl < L && pi >= pn_count) {
            ++pl;
            pi = 0;
            if (pl < L) stack_units(c, pl, U, G, pn_first, pn_count);
        }
        return pl < L;
    };
    auto issue_unit = [&]() {   // issue unit `issued` (layer pl, index pi) into its slot
        const int s = issued % kStkSlots;
        const int u = pn_first + pi, d = u / upe, j = u - d * upe, e = S.dex[pl][d];
        const uint32_t base = smem_addr(slots) + (uint32_t)s * slot_bytes;
        mbar_expect_tx(bar_gu(s), gu_unit);
        mbar_expect_tx(bar_dn(s), 10u * H);
        bulk_g2s(base, S.gu[pl] + ((size_t)e * upe + j) * gu_unit, gu_unit, bar_gu(s));
        bulk_g2s(base + gu_unit, S.dn[pl] + ((size_t)e * (I / 32) + j / 2) * 18ull * H + ((j & 1) ? 8ull * H : 0ull),
                 10u * H, bar_dn(s));
        ++issued;
        ++pi;
    };
    if (tid == 0) {
        stack_units(c, 0, U, G, pn_first, pn_count);
        for (int n = 0; n < kStkSlots && producer_next(); ++n) issue_unit();
        // x of layers 0 and 1 (layer 1's only when the layers are independent)
        for (int l = 0; l < 2 && l < L; ++l) {
            if (l == 1 && p.chained) break;
            mbar_expect_tx(bar_x(l), 2u * H);
            bulk_g2s(smem_addr(xr + (size_t)l * H), p.x + (size_t)l * H, 2u * H, bar_x(l));
        }
    }

    // ---- sum output slice of layer m (all threads) --------------------------------------
    auto reduce_layer = [&](int m) {
        const int sl = (c + m * kStkRotate) % G;
        if (sl >= H / 16) return;   // (uniform over the CTA)
        const unsigned long long t_poll = globaltimer_ns();
        if (tid == 0) {
            const unsigned long long target =
                (epoch * (unsigned long long)L + (unsigned long long)m + 1ull) * (unsigned long long)G - kDecArriveSlack;
            while ((long long)(ld_relaxed_u64(p.ctr + G) - target) < 0) {
                if (globaltimer_ns() - t_poll > p.timeout_ns) {
                    atomicOr(p.status, kDevBarrierTimeout);
                    S.abort = 1;
                    break;
                }
            }
        }
        __syncthreads();
        const bool skip = S.abort != 0;   // the same in every thread
        const int n = tid & 15, slot = tid >> 4;   // 32 slots
        constexpr int NS = kStkThreads / 16;
        constexpr int PER = (kDecMaxCtas + NS - 1) / NS;
        if (!skip) {
            const unsigned tag = stack_tag(epoch, L, m);
            const unsigned long long* col = p.part + (size_t)(m % kStkBufs) * G * H + 16 * sl + n;
            unsigned long long v[PER];
            uint32_t pending = 0;
#pragma unroll
            for (int q = 0; q < PER; ++q) {
                const int cta = slot + NS * q;
                v[q] = cta < G ? ld_relaxed_u64(col + (size_t)cta * H) : ((unsigned long long)tag << 32);
                if ((unsigned)(v[q] >> 32) != tag) pending |= 1u << q;
            }
            bool late = false;
            while (pending && !late) {
                __nanosleep(64);
#pragma unroll
                for (int q = 0; q < PER; ++q) {
                    if ((pending >> q) & 1u) {
                        v[q] = ld_relaxed_u64(col + (size_t)(slot + NS * q) * H);
                        if ((unsigned)(v[q] >> 32) == tag) pending &= ~(1u << q);
                    }
                }
                late = globaltimer_ns() - t_poll > p.timeout_ns;
            }
            float acc = 0.0f;
#pragma unroll
            for (int q = 0; q < PER; ++q) acc += __uint_as_float((uint32_t)v[q]);
            if (late) {
                atomicOr(p.status, kDevBarrierTimeout);
                S.abort = 1;
            }
            red[slot * 16 + n] = acc;
        }
        __syncthreads();
        if (tid < 16 && !skip && !S.abort) {
            float yv = 0.0f;
#pragma unroll
            for (int s2 = 0; s2 < NS; ++s2) yv += red[s2 * 16 + tid];
            reinterpret_cast<__nv_bfloat16*>(p.y + (size_t)m * H)[16 * sl + tid] = __float2bfloat16_rn(yv);
        }
        if (p.chained) __threadfence();   // the slice is visible before it is counted
        __syncthreads();
        // counted (release: this CTA's reads of the partials are done) in every launch,
        // chained or not, and on every path, so that the counts stay in lockstep with
        // the launch count; a CTA about to reuse a partial buffer waits for it
        if (tid == 0) arrive_release(p.ctr + G + 1);
    };

    // ---- the layers ---------------------------------------------------------------------
    int n = 0;              // consumer's unit sequence index
    int pending_red = -1;   // independent layers: the layer whose slice is summed next
    for (int l = 0; l < L; ++l) {
        // stage x_l as fp16 fragments with a power-of-two shift
        const uint16_t* xsrc;
        if (p.chained && l > 0) {
            // y_{l-1}, every slice of it, written by the CTAs of this launch
            if (tid == 0) {
                const unsigned long long t0 = globaltimer_ns();
                const unsigned long long target =
                    (epoch * (unsigned long long)L + (unsigned long long)l) * (unsigned long long)(H / 16);
                while ((long long)(ld_acquire_u64(p.ctr + G + 1) - target) < 0) {
                    if (globaltimer_ns() - t0 > p.timeout_ns) {
                        atomicOr(p.status, kDevBarrierTimeout);
                        S.abort = 1;
                        break;
                    }
                }
            }
            __syncthreads();
            xsrc = p.x + (size_t)l * H;   // = p.y + (l - 1) * H, read through L2 below
        } else {
            if (!mbar_wait(bar_x(l & 1), (uint32_t)(l >> 1) & 1u, p.timeout_ns) && tid == 0) {
                atomicOr(p.status, kDevLoadTimeout);
                S.abort = 1;
            }
            xsrc = xr + (size_t)(l & 1) * H;
        }
        {
            const bool global_src = p.chained && l > 0;
            float m = 0.0f;
            for (int r = tid; r < H / 2; r += kStkThreads) {
                const uint32_t two = global_src ? __ldcg(reinterpret_cast<const unsigned int*>(xsrc) + r)
                                                : reinterpret_cast<const uint32_t*>(xsrc)[r];
                m = fmaxf(m, fmaxf(fabsf(bf16_bits_to_f32((uint16_t)(two & 0xffff))),
                                   fabsf(bf16_bits_to_f32((uint16_t)(two >> 16)))));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (lane == 0) S.wmax[warp] = m;
            __syncthreads();
            float mm = 0.0f;
#pragma unroll
            for (int w2 = 0; w2 < kStkWarps; ++w2) mm = fmaxf(mm, S.wmax[w2]);
            const int sh = fp16_shift(mm);
            const float scl = pow2f(-sh);
            if (tid == 0) S.xshift = sh;
            for (int r = tid; r < H / 2; r += kStkThreads) {
                const uint32_t two = global_src ? __ldcg(reinterpret_cast<const unsigned int*>(xsrc) + r)
                                                : reinterpret_cast<const uint32_t*>(xsrc)[r];
                xs[bfrag_word(r)] = f32x2_to_f16x2_rn(bf16_bits_to_f32((uint16_t)(two & 0xffff)) * scl,
                                                      bf16_bits_to_f32((uint16_t)(two >> 16)) * scl);
            }
            __syncthreads();
        }
        // the x buffer just read takes layer l + 2's x (independent layers)
        if (tid == 0 && !p.chained && l + 2 < L) {
            mbar_expect_tx(bar_x(l & 1), 2u * H);
            bulk_g2s(smem_addr(xr + (size_t)(l & 1) * H), p.x + (size_t)(l + 2) * H, 2u * H, bar_x(l & 1));
        }
        const float xm = pow2f(S.xshift);

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
            const uint8_t* blk0 = slots + (size_t)s * slot_bytes;
            const uint8_t* blk1 = blk0 + block_bytes(H);
            // gate_up: warp w takes the 64-k quads w, w + W, ...
            float t0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, t1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            const uint32_t* brow = xs + (g == 0 ? 0 : xrw);
#pragma unroll 1
            for (int q = warp; q < nq; q += kStkWarps) {
                uint32_t b[8];
                load_bfrag(brow, q, lane, b);
                quad_mma2_b(blk0, blk1, H, b, q, lane, t0, t1);
            }
            if (c4 == 0) {   // token column 0: rows g, g + 8 of gate (t0) and up (t1)
                float* rw = red + warp * 32;
                rw[g] = t0[0];
                rw[g + 8] = t0[2];
                rw[16 + g] = t1[0];
                rw[24 + g] = t1[2];
            }
            __syncthreads();
            if (warp == 0) {
                const int half = lane >> 4, cc = lane & 15;
                float sacc = 0.0f;
#pragma unroll
                for (int w2 = 0; w2 < kStkWarps; ++w2) sacc += red[w2 * 32 + half * 16 + cc];
                const float other = __shfl_xor_sync(0xffffffffu, sacc, 16);
                const float v = half == 0 ? silu_mul_fast(sacc * xm, other * xm) * S.dw[l][d] : 0.0f;
                float mx = fabsf(v);
#pragma unroll
                for (int o = 8; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                const int sh = fp16_shift(mx);
                const float sc = pow2f(-sh);
                const float vn = __shfl_down_sync(0xffffffffu, v, 1);
                if (half == 0 && (cc & 1) == 0) S.bfrag[cc >> 1] = f32x2_to_f16x2_rn(v * sc, vn * sc);
                if (lane == 0) S.bshift = sh;
            }
            __syncthreads();
            if (!S.abort && !mbar_wait(bar_dn(s), ph, p.timeout_ns)) {
                atomicOr(p.status, kDevLoadTimeout);
                S.abort = 1;
            }
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
            __syncthreads();   // every warp is done with the slot
            if (tid == 0 && !S.abort && producer_next()) issue_unit();
            // independent layers: the previous layer's slice, now that its partials are in
            if (i == 0 && pending_red >= 0) {
                reduce_layer(pending_red);
                pending_red = -1;
            }
        }
        if (pending_red >= 0) {   // (a CTA without units in this layer)
            reduce_layer(pending_red);
            pending_red = -1;
        }
        // this CTA's partial of layer l, tagged, then one arrival.  The buffer of layer
        // l held layer l - 3, whose slices other CTAs may still be summing (a CTA that
        // sums no slice never waits for the others, so it can run ahead): wait until
        // every slice of layer l - 3 has been summed
        if (l >= kStkBufs) {
            if (tid == 0) {
                const unsigned long long t0 = globaltimer_ns();
                const unsigned long long target =
                    (epoch * (unsigned long long)L + (unsigned long long)(l - kStkBufs) + 1ull) *
                    (unsigned long long)(H / 16);
                while ((long long)(ld_acquire_u64(p.ctr + G + 1) - target) < 0) {
                    if (globaltimer_ns() - t0 > p.timeout_ns) {
                        atomicOr(p.status, kDevBarrierTimeout);
                        S.abort = 1;
                        break;
                    }
                }
            }
            __syncthreads();
        }
        if (!S.abort) {
            unsigned long long* part = p.part + ((size_t)(l % kStkBufs) * G + c) * H;
            const unsigned long long tg = (unsigned long long)stack_tag(epoch, L, l) << 32;
            if (c4 == 0) {
#pragma unroll
                for (int qs = 0; qs < kStkHQ; ++qs) {
                    const int q = warp + kStkWarps * qs;
                    if (q < nq) {
#pragma unroll
                        for (int s4 = 0; s4 < 4; ++s4) {
                            const int h0 = 16 * (4 * q + s4) + g;
                            st_relaxed_u64(part + h0, tg | __float_as_uint(Y[qs][s4][0]));
                            st_relaxed_u64(part + h0 + 8, tg | __float_as_uint(Y[qs][s4][2]));
                        }
                    }
                }
            }
        }
        __syncthreads();
        if (tid == 0) arrive_relaxed(p.ctr + G);   // once per layer on every path: lockstep counts
        if (p.chained)
            reduce_layer(l);
        else
            pending_red = l;
    }
    if (pending_red >= 0) reduce_layer(pending_red);

    // never leave with copies in flight: after an abort, wait (bounded) for the
    // last copy issued into each slot and each x buffer (phases complete in order)
    __syncthreads();
    if (tid == 0 && S.abort) {
        for (int q = issued > kStkSlots ? issued - kStkSlots : 0; q < issued; ++q) {
            const uint32_t ph = (uint32_t)(q / kStkSlots) & 1u;
            mbar_wait(bar_gu(q % kStkSlots), ph, p.timeout_ns);
            mbar_wait(bar_dn(q % kStkSlots), ph, p.timeout_ns);
        }
        const int nx = p.chained ? (L > 0 ? 1 : 0) : L;   // x copies issued: layers 0 .. nx-1
        for (int l = nx > 2 ? nx - 2 : 0; l < nx; ++l) mbar_wait(bar_x(l & 1), (uint32_t)(l >> 1) & 1u, p.timeout_ns);
    }
}

}  // namespace fe
