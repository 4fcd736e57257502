// Streaming grouped FP4 projections for moderate T (more token-expert pairs
// than the fused decode kernel takes, fewer than the tensor-core tiles want).
//
// "FireEcho Engine", sections "The Goliath Kernel: Why It's Fast" (packed
// bytes loaded, nibbles dequantised in registers, tensor-core accumulation,
// expert IDs read from device memory) and "Speed Optimization History"
// (grouped dispatch: one launch serves every routed expert, fused gate_up).
//
// One persistent CTA per SM, 8 compute warps and one producer warp.  The
// routed experts' units (gate_up: 16 gate + 16 up columns over K = H; down:
// 16 output columns over K = I) form one expert-major sequence; each CTA takes
// a contiguous range of it whose estimated cost (weight bytes, plus the MMA
// and B staging work of the expert's token blocks) is 1/grid of the total, so
// CTAs holding the units of a heavily routed expert take fewer of them (the
// ranges come from a table the grouping step fills, so a CTA reads its range
// with one load).  The
// producer streams the range through a ring of shared-memory slots with
// cp.async.bulk (a full and an empty mbarrier per slot), so copies are issued
// off the compute warps' path.  The B rows of the current expert's tokens are
// converted to fp16 with a power-of-two row shift while they are staged in
// fragment order (x rows by token for gate_up, act rows by position for down),
// and stay in shared memory for every unit of the expert the CTA holds.
//
//   gate_up: the 8 warps share each unit (a strided set of its 64-k quads
//   each); their partial sums wait in shared memory and one reduction serves
//   many units; SiLU(gate)*up goes to act (fp32, by grouped position).
//   down: one warp per unit (all its quads), so a unit's sums end in that
//   warp's registers and go straight to o (fp32, by position) for the ordered
//   combine; the warps take the units of an expert in rounds of 8.
#pragma once

#include "common.cuh"
#include "mma.cuh"

namespace fe {

constexpr int kSgComputeWarps = 8;
constexpr int kSgThreads = 32 * (kSgComputeWarps + 1);
constexpr int kSgMaxSlots = 32;
constexpr int kSgRedFloats = 4096;                                   // gate_up partials held before a reduction
constexpr int kSgMaxJobs = kSgRedFloats / (kSgComputeWarps * 32);    // act columns one reduction serves

struct SgParams {
    const uint8_t* blocks;     // gate_up: [E][I/16] units of 2 blocks; down: [E][H/16] blocks
    int K;                     // reduction length (H for gate_up, I for down)
    int n_units;               // units per expert
    uint32_t unit_bytes;       // 18K (gate_up) or 9K (down)
    int N_out;                 // row length of out (I or H)
    const int32_t* offsets;    // [E + 1] grouped positions per expert
    const int32_t* active;     // [E] routed experts, ascending
    const int32_t* n_active;   // [1]
    const int32_t* sorted_pair;
    int top_k;
    const void* bsrc;          // gate_up: x bf16 [T][H] by token; down: act fp32 [P][I] by position
    float* out;                // act [P][I] or o [P][H], by position
    uint32_t* status;
    unsigned long long timeout_ns;
    int slots;                 // ring slots (host plan)
    int chunk;                 // token rows staged at once (multiple of 8)
    const int32_t* range;      // [grid][4]: this kernel's rows of the work split table
    unsigned long long* trace;   // optional [grid][8]: clock64 at start / range known / first unit landed / end,
                                 // units, %globaltimer at start / end
};

// Byte offsets of the dynamic shared memory regions.
struct SgSmem {
    uint32_t ring, full, empty, rows, shift, pos, red, jobs, total;
};

__host__ __device__ inline SgSmem sg_smem_layout(bool gate_up, int K, uint32_t unit_bytes, int slots, int chunk)
{
    SgSmem L;
    L.ring = 0;
    L.full = (uint32_t)slots * unit_bytes;
    L.empty = L.full + 8u * slots;
    L.rows = (L.empty + 8u * slots + 15u) & ~15u;
    L.shift = L.rows + 4u * (uint32_t)(chunk + 1) * (uint32_t)brow_words(K);
    L.pos = L.shift + 4u * (uint32_t)chunk;
    L.red = (L.pos + 4u * (uint32_t)chunk + 15u) & ~15u;
    L.jobs = L.red + (gate_up ? 4u * kSgRedFloats : 0u);
    L.total = L.jobs + (gate_up ? 16u * kSgMaxJobs : 0u);
    return L;
}

struct SgShared {
    int a0, j0, nu;   // first unit (active index, unit) and unit count of this CTA
    int issued;       // units the producer issued
    int abort;
};

FE_DEV uint32_t sg_smem(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

FE_DEV void sg_bar_compute() { asm volatile("bar.sync 1, %0;" ::"n"(32 * kSgComputeWarps) : "memory"); }

// Bounded wait for phase `parity` (test_wait polling: no suspension past the
// completion, which try_wait was seen to add).
FE_DEV bool sg_wait(uint32_t bar, uint32_t parity, unsigned long long timeout_ns)
{
    uint32_t ok = 0;
    unsigned long long t0 = 0;
    for (int it = 0;; ++it) {
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(bar), "r"(parity)
            : "memory");
        if (ok) return true;
        if (it == 0) t0 = globaltimer_ns();
        else if ((it & 15) == 0 && globaltimer_ns() - t0 > timeout_ns) return false;
    }
}

FE_DEV void sg_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// A fragments and group-scale words of quad q of one fragment-ordered block
// (16 columns x K): four k16 steps of four f16x2 registers.
FE_DEV void sg_quad_a(const uint8_t* blk, int K, int q, int lane, uint32_t (&a)[4][4], uint32_t (&sw)[2])
{
    const int g = lane >> 2;
    const uint4 cw = *reinterpret_cast<const uint4*>(blk + 512 * q + 16 * lane);
    e2m1x8_to_f16x2x4(cw.x, a[0]);
    e2m1x8_to_f16x2x4(cw.y, a[1]);
    e2m1x8_to_f16x2x4(cw.z, a[2]);
    e2m1x8_to_f16x2x4(cw.w, a[3]);
#pragma unroll
    for (int gi = 0; gi < 2; ++gi) sw[gi] = *reinterpret_cast<const uint32_t*>(blk + 8 * K + 4 * ((2 * q + gi) * 8 + g));
}

// tot += (A . B) of one quad, the bf16 group scale applied to each 32-k half.
FE_DEV void sg_quad_mma(const uint32_t (&a)[4][4], const uint32_t (&sw)[2], const uint32_t (&b)[8], float* tot)
{
#pragma unroll
    for (int gi = 0; gi < 2; ++gi) {
        float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        mma16816(d, a[2 * gi], b[4 * gi], b[4 * gi + 1]);
        mma16816(d, a[2 * gi + 1], b[4 * gi + 2], b[4 * gi + 3]);
        const float slo = __uint_as_float(sw[gi] << 16), shi = __uint_as_float(sw[gi] & 0xffff0000u);
        tot[0] = fmaf(d[0], slo, tot[0]);
        tot[1] = fmaf(d[1], slo, tot[1]);
        tot[2] = fmaf(d[2], shi, tot[2]);
        tot[3] = fmaf(d[3], shi, tot[3]);
    }
}

// Work split of the two streaming kernels, computed once by the grouping's
// single-CTA step (which has the counts at hand): for each kernel and CTA c,
// the contiguous range of the expert-major unit sequence whose units start
// (in cumulative cost) within [c * total / G, (c + 1) * total / G).
struct SgSplit {
    int32_t* table;   // [2][G][4]: first active index, first unit, unit count, 0 (gate_up, then down)
    int G;
    int n_units[2], chunk[2], c_bytes[2], c_chunk[2], c_block[2], c_restage[2];
};

FE_DEV long long sg_split_cost(const SgSplit& s, int ph, int npos)
{
    const int nb = (npos + 7) / 8, nc = (npos + s.chunk[ph] - 1) / s.chunk[ph];
    const int c = s.c_chunk[ph] * nc + s.c_block[ph] * nb + (nc > 1 ? s.c_restage[ph] * nc : 0);
    return (long long)max(s.c_bytes[ph], c) * s.n_units[ph];
}

// Whole CTA.  counts (per expert), active and na are visible to every thread;
// scratch holds 2 (na + 1) + 32 long longs.
FE_DEV void sg_plan_ranges(const SgSplit& s, const int32_t* counts, const int32_t* active, int na, long long* scratch)
{
    const int nthreads = blockDim.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    long long* pre = scratch;                 // [2][na + 1] cumulative cost before active expert a
    long long* wsum = scratch + 2 * (na + 1); // [32] per-warp totals
    const int per = (na + nthreads - 1) / nthreads, a0 = tid * per;
    for (int ph = 0; ph < 2; ++ph) {
        long long loc = 0;
        for (int a = a0; a < a0 + per && a < na; ++a) loc += sg_split_cost(s, ph, counts[active[a]]);
        long long incl = loc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        long long base = 0;
        for (int w = 0; w < warp; ++w) base += wsum[w];
        long long run = base + incl - loc;
        for (int a = a0; a < a0 + per && a < na; ++a) {
            pre[ph * (na + 1) + a] = run;
            run += sg_split_cost(s, ph, counts[active[a]]);
        }
        if (a0 < na && a0 + per >= na) pre[ph * (na + 1) + na] = run;
        if (na == 0 && tid == 0) pre[ph * (na + 1)] = 0;
        __syncthreads();
    }
    // one thread per (kernel, CTA): binary searches for its two bounds
    for (int i = tid; i < 2 * s.G; i += nthreads) {
        const int ph = i / s.G, c = i - ph * s.G;
        const long long* pr = pre + ph * (na + 1);
        const long long total = pr[na];
        int bound[2][2];
        for (int side = 0; side < 2; ++side) {
            const long long t = total * (c + side) / s.G;
            int a = na, j = 0;
            if (t < total) {
                int lo = 0, hi = na - 1;   // the last a with pr[a] <= t
                while (lo < hi) {
                    const int mid = (lo + hi + 1) >> 1;
                    if (pr[mid] <= t) lo = mid;
                    else hi = mid - 1;
                }
                a = lo;
                const long long cu = (pr[a + 1] - pr[a]) / s.n_units[ph];   // cost of one unit
                j = (int)((t - pr[a] + cu - 1) / cu);
                if (j >= s.n_units[ph]) {
                    a += 1;
                    j = 0;
                }
            }
            bound[side][0] = a;
            bound[side][1] = j;
        }
        const long long u0 = (long long)bound[0][0] * s.n_units[ph] + bound[0][1];
        const long long u1 = (long long)bound[1][0] * s.n_units[ph] + bound[1][1];
        int32_t* row = s.table + 4 * (size_t)i;
        row[0] = bound[0][0];
        row[1] = bound[0][1];
        row[2] = (int)max(0ll, u1 - u0);
        row[3] = 0;
    }
}

// Stage cnt B rows (positions pos0 ..) into shared memory as fp16 pairs in
// fragment order, each scaled by 2^-s with s = fp16_shift(row max); one
// compute warp per row.  BF16: x rows by token (bf16); otherwise act rows by
// position (fp32).
template <bool BF16>
FE_DEV void sg_stage_rows(const SgParams& p, int pos0, int cnt, uint32_t* rows, int* shift, int* posr, int warp,
                          int lane)
{
    const int K = p.K, rw = brow_words(K);
    for (int r = warp; r < cnt; r += kSgComputeWarps) {
        const int pos = pos0 + r;
        const int src = BF16 ? p.sorted_pair[pos] / p.top_k : pos;
        float m = 0.0f;
        if (BF16) {
            const uint4* row = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.bsrc) + (size_t)src * K);
            for (int i = lane; i < K / 8; i += 32) {
                const uint4 v = __ldg(row + i);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int t = 0; t < 4; ++t)
                    m = fmaxf(m, fmaxf(fabsf(bf16_bits_to_f32((uint16_t)(w[t] & 0xffffu))),
                                       fabsf(bf16_bits_to_f32((uint16_t)(w[t] >> 16)))));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            const int sh = fp16_shift(m);
            const float sc = pow2f(-sh);
            for (int i = lane; i < K / 8; i += 32) {
                const uint4 v = __ldg(row + i);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int t = 0; t < 4; ++t)
                    rows[r * rw + bfrag_word((uint32_t)(4 * i + t))] =
                        f32x2_to_f16x2_rn(bf16_bits_to_f32((uint16_t)(w[t] & 0xffffu)) * sc,
                                          bf16_bits_to_f32((uint16_t)(w[t] >> 16)) * sc);
            }
            if (lane == 0) shift[r] = sh;
        } else {
            const float4* row = reinterpret_cast<const float4*>(static_cast<const float*>(p.bsrc) + (size_t)src * K);
            for (int i = lane; i < K / 4; i += 32) {
                const float4 v = __ldg(row + i);
                m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            const int sh = fp16_shift(m);
            const float sc = pow2f(-sh);
            for (int i = lane; i < K / 4; i += 32) {
                const float4 v = __ldg(row + i);
                rows[r * rw + bfrag_word((uint32_t)(2 * i))] = f32x2_to_f16x2_rn(v.x * sc, v.y * sc);
                rows[r * rw + bfrag_word((uint32_t)(2 * i + 1))] = f32x2_to_f16x2_rn(v.z * sc, v.w * sc);
            }
            if (lane == 0) shift[r] = sh;
        }
        if (lane == 0) posr[r] = pos;
    }
}

// NB: 8-token blocks per staged chunk at most (p.chunk <= 8 NB).
template <bool GATE_UP, int NB>
__global__ void __launch_bounds__(kSgThreads, 1) sg_kernel(SgParams p)
{
    extern __shared__ __align__(128) uint8_t sg_sm[];
    __shared__ SgShared S;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g = lane >> 2;
    const int K = p.K, rw = brow_words(K), C = p.chunk, R = p.slots;
    constexpr int UB = 1;   // units per copy batch (one full barrier per batch); R is a multiple of UB
    const SgSmem L = sg_smem_layout(GATE_UP, K, p.unit_bytes, R, C);
    uint8_t* ring = sg_sm + L.ring;
    const uint32_t full0 = sg_smem(sg_sm + L.full), empty0 = sg_smem(sg_sm + L.empty);
    uint32_t* rows = reinterpret_cast<uint32_t*>(sg_sm + L.rows);
    int* shift = reinterpret_cast<int*>(sg_sm + L.shift);
    int* posr = reinterpret_cast<int*>(sg_sm + L.pos);

    if (tid < R) {
        if (tid < R / UB) asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(full0 + 8 * tid) : "memory");
        asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(empty0 + 8 * tid), "r"(GATE_UP ? kSgComputeWarps : 1)
                     : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");   // each initialising thread
    }
    if (tid == 0) {
        S.abort = 0;
        S.issued = 0;
    }
    for (int i = tid; i < rw; i += kSgThreads) rows[C * rw + i] = 0u;   // the zero row
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    unsigned long long* tr = p.trace ? p.trace + (size_t)blockIdx.x * 8 : nullptr;
    if (tr && tid == 0) {
        tr[0] = (unsigned long long)clock64();
        tr[5] = globaltimer_ns();
    }
    if (tid == 0) {
        const int4 r = *reinterpret_cast<const int4*>(p.range + 4 * blockIdx.x);
        S.a0 = r.x;
        S.j0 = r.y;
        S.nu = r.z;
    }
    __syncthreads();
    const int nu = S.nu;
    if (tr && tid == 0) {
        tr[1] = (unsigned long long)clock64();
        tr[4] = (unsigned long long)nu;
    }
    if (nu == 0) return;

    if (warp == kSgComputeWarps) {
        // ---- producer: the range's units into the ring as slots free up, in the
        // order the compute warps take them (gate_up: one pass over an expert's
        // units per chunk of its token rows).  The walk is written for batches of
        // UB units (one full barrier per batch, runs of consecutive units of an
        // expert as one copy, one empty barrier per unit); UB is 1, one copy and
        // one full barrier per unit, since 8-unit batches of down units made a
        // wait time out (cause not found).  Every lane walks the same sequence;
        // lane l takes the l-th unit of each batch and waits for its slot. ---------
        int a = S.a0, j = S.j0, left = nu, ch = 0, seg_i = 0, pu = 0;
        int seg_n = 0, passes = 1, e = 0;
        auto enter_segment = [&]() {
            e = p.active[a];
            const int npos = p.offsets[e + 1] - p.offsets[e];
            seg_n = min(left, p.n_units - j);
            passes = GATE_UP ? (npos + C - 1) / C : 1;
            ch = 0;
            seg_i = 0;
        };
        enter_segment();
        bool stop = false;
        while (left > 0 && !stop) {
            int my_e = -1, my_j = 0;
            int nb = 0;
            for (; nb < UB && left > 0; ++nb) {
                if (nb == lane) {
                    my_e = e;
                    my_j = j + seg_i;
                }
                if (++seg_i == seg_n) {
                    seg_i = 0;
                    if (++ch == passes) {
                        left -= seg_n;
                        j += seg_n;
                        if (j == p.n_units) {
                            j = 0;
                            ++a;
                        }
                        if (left > 0) enter_segment();
                    }
                }
            }
            // every unit's slot free first (a unit waits for the one R before it)
            bool ok = true;
            const int x = pu + lane, slot = x % R;
            if (lane < nb && x >= R)
                ok = !*reinterpret_cast<volatile int*>(&S.abort) &&
                     sg_wait(empty0 + 8 * slot, (uint32_t)((x / R - 1) & 1), p.timeout_ns);
            if (__ballot_sync(0xffffffffu, !ok)) {
                if (lane == 0) {
                    if (!S.abort) atomicOr(p.status, 0x8u);
                    S.abort = 1;
                }
                break;
            }
            const int bi = pu / UB;   // batch index
            const uint32_t bar = full0 + 8 * (bi % (R / UB));
            if (lane == 0)
                asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"((uint32_t)nb * p.unit_bytes)
                             : "memory");
            __syncwarp();
            // runs of consecutive units of one expert: one copy each, from the run's first lane
            const int pe = __shfl_up_sync(0xffffffffu, my_e, 1), pj = __shfl_up_sync(0xffffffffu, my_j, 1);
            const bool start = lane < nb && (lane == 0 || pe != my_e || pj + 1 != my_j);
            const unsigned starts = __ballot_sync(0xffffffffu, start) | (nb < 32 ? (1u << nb) : 0u);
            if (start) {
                const unsigned later = starts & ~((2u << lane) - 1u);
                const int run = __ffs(later) - 1 - lane;
                asm volatile(
                    "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                        sg_smem(ring + (size_t)slot * p.unit_bytes)),
                    "l"(p.blocks + ((size_t)my_e * p.n_units + my_j) * p.unit_bytes), "r"((uint32_t)run * p.unit_bytes),
                    "r"(bar)
                    : "memory");
            }
            pu += nb;
        }
        if (lane == 0) S.issued = pu;
    } else if (GATE_UP) {
        // ---- gate_up: all compute warps on each unit, deferred reductions ---------------
        const int nq = K / 64;
        float* red = reinterpret_cast<float*>(sg_sm + L.red);
        int* jobs = reinterpret_cast<int*>(sg_sm + L.jobs);   // [kSgMaxJobs][4]: act offset, red base, stride, shift
        int njobs = 0, red_used = 0;   // the same in every compute thread
        auto flush = [&]() {
            sg_bar_compute();
            if (!*reinterpret_cast<volatile int*>(&S.abort)) {
                const int half = lane & 1, n = lane >> 1;
                for (int jb = warp; jb < njobs; jb += kSgComputeWarps) {
                    const int* jr = jobs + 4 * jb;
                    const float* rwp = red + jr[1] + half * (kSgComputeWarps / 2) * jr[2] + n;
                    float gs = 0.0f, us = 0.0f;
#pragma unroll
                    for (int w2 = 0; w2 < kSgComputeWarps / 2; ++w2) {
                        gs += rwp[w2 * jr[2]];
                        us += rwp[w2 * jr[2] + 16];
                    }
                    gs += __shfl_xor_sync(0xffffffffu, gs, 1);
                    us += __shfl_xor_sync(0xffffffffu, us, 1);
                    if (half == 0) {
                        const float m = pow2f(jr[3]);
                        p.out[(size_t)jr[0] + n] = silu_mul_fast(gs * m, us * m);
                    }
                }
            }
            sg_bar_compute();
            njobs = 0;
            red_used = 0;
        };
        int ca = S.a0, cj0 = S.j0, left = nu, vu = 0;
        while (left > 0) {
            const int e = p.active[ca];
            const int pos0 = p.offsets[e], npos = p.offsets[e + 1] - pos0;
            const int seg_n = min(left, p.n_units - cj0);
            const int nch = (npos + C - 1) / C;
            for (int ch = 0; ch < nch; ++ch) {
                const int cnt = min(C, npos - ch * C);
                // the chunk's rows, once per pass over the expert's units; pending jobs
                // keep their own offsets and shifts, and nobody reads the old rows once
                // every compute warp is here
                sg_bar_compute();
                sg_stage_rows<true>(p, pos0 + ch * C, cnt, rows, shift, posr, warp, lane);
                sg_bar_compute();
                const int nblk = (cnt + 7) / 8;
                for (int i = 0; i < seg_n; ++i, ++vu) {
                    const int slot = vu % R, cj = cj0 + i;
                    const uint8_t* blk0 = ring + (size_t)slot * p.unit_bytes;
                    const uint8_t* blk1 = blk0 + block_bytes(K);
                    if (!*reinterpret_cast<volatile int*>(&S.abort) &&
                        !sg_wait(full0 + 8 * ((vu / UB) % (R / UB)), (uint32_t)(((vu / UB) / (R / UB)) & 1), p.timeout_ns)) {
                        atomicOr(p.status, 0x8u);
                        S.abort = 1;
                    }
                    if (tr && tid == 0 && vu == 0) tr[2] = (unsigned long long)clock64();
                    const int need = kSgComputeWarps * cnt * 32;
                    if (red_used + need > kSgRedFloats || njobs + cnt > kSgMaxJobs) flush();
                    float acc[NB][8];
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                        for (int t = 0; t < 8; ++t) acc[nb][t] = 0.0f;
                    for (int q = warp; q < nq; q += kSgComputeWarps) {
                        uint32_t a0[4][4], s0[2], a1[4][4], s1[2];
                        sg_quad_a(blk0, K, q, lane, a0, s0);
                        sg_quad_a(blk1, K, q, lane, a1, s1);
#pragma unroll
                        for (int nb = 0; nb < NB; ++nb) {
                            if (nb < nblk) {
                                const int r = 8 * nb + g;
                                uint32_t b[8];
                                load_bfrag(rows + (r < cnt ? r : C) * rw, q, lane, b);
                                sg_quad_mma(a0, s0, b, &acc[nb][0]);
                                sg_quad_mma(a1, s1, b, &acc[nb][4]);
                            }
                        }
                    }
                    // this warp is done reading the unit's slot
                    __syncwarp();
                    if (lane == 0) sg_arrive(empty0 + 8 * slot);
                    // partials of the valid token columns: [warp][column][gate 16 | up 16];
                    // lane (g, c) holds rows g, g+8 of columns 2c, 2c+1 of each block
                    {
                        const int c = lane & 3;
                        float* rwb = red + red_used + warp * cnt * 32;
#pragma unroll
                        for (int nb = 0; nb < NB; ++nb) {
                            if (nb < nblk) {
#pragma unroll
                                for (int e2 = 0; e2 < 2; ++e2) {
                                    const int jc = 8 * nb + 2 * c + e2;
                                    if (jc < cnt) {
                                        float* rwp = rwb + jc * 32;
                                        rwp[g] = acc[nb][e2];
                                        rwp[g + 8] = acc[nb][2 + e2];
                                        rwp[16 + g] = acc[nb][4 + e2];
                                        rwp[24 + g] = acc[nb][6 + e2];
                                    }
                                }
                            }
                        }
                    }
                    if (tid < cnt) {
                        int* jr = jobs + 4 * (njobs + tid);
                        jr[0] = posr[tid] * p.N_out + 16 * cj;
                        jr[1] = red_used + tid * 32;
                        jr[2] = cnt * 32;
                        jr[3] = shift[tid];
                    }
                    njobs += cnt;
                    red_used += need;
                }
            }
            left -= seg_n;
            cj0 += seg_n;
            if (cj0 == p.n_units) {
                cj0 = 0;
                ++ca;
            }
        }
        flush();
    } else {
        // ---- down: one warp per unit, rounds of 8 units within an expert ------------------
        const int nq = K / 64;
        int ca = S.a0, cj = S.j0;   // consumer cursor at the start of a segment
        int u = 0;
        while (u < nu) {
            const int e = p.active[ca];
            const int pos0 = p.offsets[e], npos = p.offsets[e + 1] - pos0;
            const int seg_n = min(nu - u, p.n_units - cj);   // this expert's units in the range
            const int nch = (npos + C - 1) / C;
            for (int rb = 0; rb < seg_n; rb += kSgComputeWarps) {
                // the warps meet between rounds, so that no warp waits on a full
                // barrier while the batch that used it two phases ago is still in
                // flight (a parity wait cannot tell those phases apart); the
                // staging below meets anyway
                if (rb > 0 && nch == 1) sg_bar_compute();
                const int my = rb + warp;   // this warp's unit of the round
                const bool have = my < seg_n;
                const int uu = u + my, slot = uu % R, unit = cj + my;
                for (int ch = 0; ch < nch; ++ch) {
                    const int cnt = min(C, npos - ch * C);
                    if (nch > 1 || (rb == 0 && ch == 0)) {
                        sg_bar_compute();
                        sg_stage_rows<false>(p, pos0 + ch * C, cnt, rows, shift, posr, warp, lane);
                        sg_bar_compute();
                    }
                    if (!have) continue;
                    if (ch == 0 && !*reinterpret_cast<volatile int*>(&S.abort) &&
                        !sg_wait(full0 + 8 * ((uu / UB) % (R / UB)), (uint32_t)(((uu / UB) / (R / UB)) & 1), p.timeout_ns)) {
                        atomicOr(p.status, 0x8u);
                        S.abort = 1;
                    }
                    if (tr && lane == 0 && uu == 0 && ch == 0) tr[2] = (unsigned long long)clock64();
                    if (*reinterpret_cast<volatile int*>(&S.abort)) continue;
                    const uint8_t* blk = ring + (size_t)slot * p.unit_bytes;
                    const int nblk = (cnt + 7) / 8;
                    float acc[NB][4];
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                        for (int i = 0; i < 4; ++i) acc[nb][i] = 0.0f;
#pragma unroll 2
                    for (int q = 0; q < nq; ++q) {
                        uint32_t a0[4][4], s0[2];
                        sg_quad_a(blk, K, q, lane, a0, s0);
#pragma unroll
                        for (int nb = 0; nb < NB; ++nb) {
                            if (nb < nblk) {
                                const int r = 8 * nb + g;
                                uint32_t b[8];
                                load_bfrag(rows + (r < cnt ? r : C) * rw, q, lane, b);
                                sg_quad_mma(a0, s0, b, &acc[nb][0]);
                            }
                        }
                    }
                    // lane (g, c): outputs g, g+8 of token columns 2c, 2c+1 of each block
                    const int c = lane & 3;
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb) {
                        if (nb < nblk) {
#pragma unroll
                            for (int e2 = 0; e2 < 2; ++e2) {
                                const int jc = 8 * nb + 2 * c + e2;
                                if (jc < cnt) {
                                    const float m = pow2f(shift[jc]);
                                    float* o = p.out + (size_t)posr[jc] * p.N_out + 16 * unit;
                                    o[g] = acc[nb][e2] * m;
                                    o[g + 8] = acc[nb][2 + e2] * m;
                                }
                            }
                        }
                    }
                }
                if (have) {
                    __syncwarp();
                    if (lane == 0) sg_arrive(empty0 + 8 * slot);
                }
            }
            u += seg_n;
            cj += seg_n;
            if (cj == p.n_units) {
                cj = 0;
                ++ca;
            }
        }
    }
    if (tr && tid == 0) {
        tr[3] = (unsigned long long)clock64();
        tr[6] = globaltimer_ns();
    }
    // never leave with copies in flight: after an abort, wait (bounded) for the
    // last unit issued into each slot
    __syncthreads();
    if (S.abort && tid == 0) {
        const int issued = S.issued;
        for (int x = max(0, issued - R); x < issued; x += UB)
            sg_wait(full0 + 8 * ((x / UB) % (R / UB)), (uint32_t)(((x / UB) / (R / UB)) & 1), p.timeout_ns);
    }
}

}  // namespace fe
