// Fused small-T decode layer: one launch per layer.
//
// "FireEcho Engine", sections "Speed Optimization History" (single-token
// decode fast path, multi-expert kernel, packed contiguous expert buffer,
// CUDA-graph decode) and "The Goliath Kernel: Why It's Fast" (expert IDs read
// on the GPU, FP4 dequantised in registers, nothing dequantised written to
// memory).  The pages' kernel runs one Triton launch per projection; here the
// whole layer is one launch, so that the HBM stream of the down weights
// overlaps the gate_up work and no launch boundary sits inside the layer:
//
//   1. one bulk copy brings the T router-logit rows and the T x rows into
//      shared memory; every CTA routes the T tokens itself (the rank of each
//      logit among the E logits of its token, counted by all threads in
//      parallel: rank < k selects it as slot rank, ties to the lower index)
//      and groups the T*k pairs by expert; CTA 0 also publishes the routing;
//   2. from the routed experts every CTA looks up its contiguous range of
//      units in a work-split table computed at reserve time: the gate_up units
//      (expert, column tile) and the down units (16-column h-slice over all
//      routed experts), cut into per-CTA ranges of equal bytes;
//   3. one thread issues cp.async.bulk copies of ALL the CTA's weight bytes
//      (both phases) into shared memory at once, one mbarrier per unit;
//   4. gate_up units are reduced over K as soon as their bytes land, SwiGLU
//      applied, act written to global memory (L2) as 64-bit words holding
//      the fp32 value and the launch's epoch tag;
//   5. each CTA that owns down units reads act back, polling (bounded) until
//      every word carries this launch's tag -- the data is its own ready
//      flag, so no grid-wide barrier round trip is needed;
//   6. each CTA computes the 16 output columns of its h-slices for every
//      pair from the down bytes already in shared memory and combines them in
//      slot order: y is written once, without atomics.
//
// The kernel is launched with programmatic dependent launch: its CTAs load
// only static data before griddepcontrol.wait, so the next layer's CTAs can
// be resident and waiting while this layer finishes.
#pragma once

#include "common.cuh"

namespace fe {

constexpr int kDecThreads = 256;
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
    const uint8_t* gu_tiles;  // [E][gu_ntiles] tiles of gu_tile_bytes
    int gu_ntiles;
    uint32_t gu_tile_bytes;
    const uint8_t* dn_tiles;  // [E][H/16] tiles of dn_tile_bytes
    uint32_t dn_tile_bytes;
    const int32_t* plan_first;  // [kDecMaxPairs + 1][grid + 1] first unit of each CTA, per nd
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

// ---- work split (host: table construction; the kernel only reads the table) ----
struct DecodePlan {
    int64_t gu_bytes, dn_bytes, total;
    int n_gu, n_dn, grid;
};

inline DecodePlan decode_plan(int nd, int H, uint32_t gu_tile_bytes, int gu_ntiles, uint32_t dn_tile_bytes, int grid)
{
    DecodePlan p;
    p.gu_bytes = gu_tile_bytes;
    p.dn_bytes = (int64_t)nd * dn_tile_bytes;
    p.n_gu = nd * gu_ntiles;
    p.n_dn = H / 16;
    p.total = p.n_gu * p.gu_bytes + p.n_dn * p.dn_bytes;
    p.grid = grid;
    return p;
}

inline int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }

// First unit of CTA c: units are laid end to end in byte order (gate_up units,
// then down units) and CTA c takes those whose first byte falls in
// [c * total / grid, (c + 1) * total / grid).
inline int decode_first_unit(const DecodePlan& p, int c)
{
    const int64_t t0 = (int64_t)c * p.total;
    const int64_t gu_end = (int64_t)p.n_gu * p.gu_bytes;
    if (t0 <= gu_end * p.grid) {
        const int64_t i = ceil_div64(t0, (int64_t)p.grid * p.gu_bytes);
        return (int)(i < p.n_gu ? i : p.n_gu);
    }
    const int64_t j = ceil_div64(t0 - gu_end * p.grid, (int64_t)p.grid * p.dn_bytes);
    return p.n_gu + (int)(j < p.n_dn ? j : p.n_dn);
}

inline int64_t decode_unit_bytes(const DecodePlan& p, int u) { return u < p.n_gu ? p.gu_bytes : p.dn_bytes; }

// ---- PTX wrappers --------------------------------------------------------------
FE_DEV uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

FE_DEV unsigned long long globaltimer()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

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
    const unsigned long long t0 = globaltimer();
    for (;;) {
        if (mbar_try_wait(bar, 0)) return true;
        if (globaltimer() - t0 > timeout_ns) return false;
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

// Reduce 16 per-lane values over the 32/C lanes that share lane % C
// (butterfly reduce-scatter): afterwards this lane holds NOUT = max(1, 16C/32)
// finished sums, for columns col0 .. col0 + NOUT - 1 of its chunk.
template <int C>
struct Butterfly {
    static constexpr int L = 32 / C;
    static constexpr int NOUT = (16 / L) > 0 ? (16 / L) : 1;
};

template <int C>
FE_DEV int butterfly16(float (&v)[16], int lane)
{
    int col0 = 0;
    int n = 16;
#pragma unroll
    for (int m = 16; m >= C; m >>= 1) {
        if (n > 1) {
            const int half = n >> 1;
            const bool up = (lane & m) != 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (j < half) {
                    const float send = up ? v[j] : v[j + half];
                    const float keep = up ? v[j + half] : v[j];
                    v[j] = keep + __shfl_xor_sync(0xffffffffu, send, m);
                }
            }
            if (up) col0 += half;
            n = half;
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], m);
        }
    }
    return col0;
}

// Padded f16x2 row index: one spare word per 16 rows (bank spread).
FE_DEV int padrow(int r) { return r + (r >> 4); }
__host__ __device__ inline int padded_rows(int rows) { return rows + rows / 16 + 1; }

// Power-of-two shift s >= 0 with m * 2^-s < 2^15 (m = max |v| of a row).
FE_DEV int fp16_shift(float m)
{
    int s = 0;
    if (m >= 32768.0f && m <= 3.0e38f) s = (int)((__float_as_uint(m) >> 23) & 0xff) - 127 - 14;
    return s;
}

FE_DEV float pow2f(int e) { return __uint_as_float((uint32_t)(127 + e) << 23); }

FE_DEV float logit_key(float v) { return v != v ? -INFINITY : v; }

struct DecodeShared {
    int sel_e[kDecMaxPairs];
    float sel_w[kDecMaxPairs];
    int sp[kDecMaxPairs];         // pair ids in (expert, pair) order
    int pdi[kDecMaxPairs];        // pair -> distinct-expert index
    int dex[kDecMaxPairs];        // distinct experts, ascending
    int dstart[kDecMaxPairs + 1]; // first sorted position of each distinct expert
    int pf0[kDecMaxPairs + 1];    // this CTA's first unit, per nd
    int pf1[kDecMaxPairs + 1];    // the next CTA's first unit, per nd
    int xshift[kDecMaxPairs];
    int ashift[kDecMaxPairs];
    int nd;
    int abort;
    unsigned tag;
    float wmax[kDecWarps];
    float ob[kDecMaxPairs * 16];  // down: [pair][16] outputs
};

// Byte offsets of the dynamic shared memory regions.
struct DecodeSmem {
    uint32_t mbar, shared, red, xs, as, lg, xr, total;
};

__host__ __device__ inline uint32_t align16(uint32_t v) { return (v + 15u) & ~15u; }

__host__ __device__ inline DecodeSmem decode_smem_layout(uint32_t weight_bytes, int T, int k, int H, int I, int E, int TW)
{
    DecodeSmem L;
    L.mbar = weight_bytes;
    L.shared = L.mbar + 8 * (kDecMaxItems + 1);
    L.red = align16(L.shared + (uint32_t)sizeof(DecodeShared));
    L.xs = L.red + 4u * kDecWarps * TW;
    L.as = L.xs + 4u * T * padded_rows(H / 2);
    L.lg = align16(L.as + 4u * T * k * padded_rows(I / 2));
    L.xr = align16(L.lg + 4u * T * E);
    L.total = align16(L.xr + 2u * T * H);
    return L;
}

template <int C>
__global__ void __launch_bounds__(kDecThreads, 1) decode_kernel(DecodeParams p)
{
    extern __shared__ __align__(128) uint8_t dsm[];
    constexpr int TW = 16 * C;
    constexpr int TN = TW / 2;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int T = p.T, E = p.E, H = p.H, I = p.I, k = p.k, P = T * k;
    const int G = H / 32, Gd = I / 32;
    const DecodeSmem L = decode_smem_layout(p.weight_bytes, T, k, H, I, E, TW);

    uint8_t* wbuf = dsm;
    DecodeShared& S = *reinterpret_cast<DecodeShared*>(dsm + L.shared);
    float* red = reinterpret_cast<float*>(dsm + L.red);
    uint32_t* xs = reinterpret_cast<uint32_t*>(dsm + L.xs);
    uint32_t* as = reinterpret_cast<uint32_t*>(dsm + L.as);
    float* lg = reinterpret_cast<float*>(dsm + L.lg);
    uint16_t* xr = reinterpret_cast<uint16_t*>(dsm + L.xr);
    const int xrow = padded_rows(H / 2), arow = padded_rows(I / 2);
    const uint32_t mbar0 = smem_addr(dsm + L.mbar);
    const uint32_t in_bar = mbar0 + 8 * kDecMaxItems;
    const bool tracing = p.trace != nullptr;
    unsigned long long* trace = tracing ? p.trace + (size_t)blockIdx.x * 16 : nullptr;
    if (tracing && tid == 0) trace[0] = globaltimer();

    // ---- 0. static data only, then wait for the previous grid ---------------------
    if (tid <= kDecMaxPairs) {
        S.pf0[tid] = p.plan_first[tid * (gridDim.x + 1) + blockIdx.x];
        S.pf1[tid] = p.plan_first[tid * (gridDim.x + 1) + blockIdx.x + 1];
    }
    if (tid == 0) {
        mbar_init(in_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        S.abort = 0;
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (tid == 0) {
        // this launch's epoch tag; the last CTA to read it advances it
        const unsigned e0 = ld_acquire_gpu(p.sync + 1);
        const unsigned arrived = atomicAdd(p.sync, 1u);
        const unsigned tag = (e0 + 1u) ? (e0 + 1u) : 1u;
        S.tag = tag;
        if (arrived == gridDim.x - 1) {
            // every CTA has read the epoch: advance it for the next launch
            atomicExch(p.sync, 0u);
            st_release_gpu(p.sync + 1, tag);
        }
        if (p.bulk_inputs) {
            const uint32_t lb = 4u * T * E, xb = 2u * T * H;
            mbar_expect_tx(in_bar, lb + xb);
            bulk_g2s(smem_addr(lg), p.logits, lb, in_bar);
            bulk_g2s(smem_addr(xr), p.x, xb, in_bar);
        }
    }
    if (!p.bulk_inputs) {
        for (int i = tid; i < T * E; i += kDecThreads) lg[i] = p.logits[i];
        for (int i = tid; i < T * H; i += kDecThreads) xr[i] = p.x[i];
    }
    __syncthreads();
    if (p.bulk_inputs && !mbar_wait0(in_bar, p.timeout_ns)) {
        if (tid == 0) atomicOr(p.status, kDevLoadTimeout);
        return;   // the copies never completed: nothing can be in flight any more
    }
    if (tracing && tid == 0) trace[8] = globaltimer();

    // ---- 1. routing: rank of every logit among its token's E logits ------------------
    bool nan_seen = false;
    for (int t = 0; t < T; ++t) {
        const float* row = lg + t * E;
        for (int e = tid; e < E; e += kDecThreads) {
            const float v = logit_key(row[e]);
            nan_seen |= row[e] != row[e];
            int rank = 0;
            int e2 = 0;
            if ((E & 3) == 0) for (; e2 + 4 <= E; e2 += 4) {
                const float4 o = *reinterpret_cast<const float4*>(row + e2);
                const float o0 = logit_key(o.x), o1 = logit_key(o.y), o2 = logit_key(o.z), o3 = logit_key(o.w);
                rank += (o0 > v) || (o0 == v && e2 < e);
                rank += (o1 > v) || (o1 == v && e2 + 1 < e);
                rank += (o2 > v) || (o2 == v && e2 + 2 < e);
                rank += (o3 > v) || (o3 == v && e2 + 3 < e);
            }
            for (; e2 < E; ++e2) {
                const float o = logit_key(row[e2]);
                rank += (o > v) || (o == v && e2 < e);
            }
            if (rank < k) {
                S.sel_e[t * k + rank] = e;
                S.sel_w[t * k + rank] = v;
            }
        }
    }
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

    // ---- 2. grouping (warp 0): stable order by expert --------------------------
    if (warp == 0) {
        const int ep = lane < P ? S.sel_e[lane] : 0x7fffffff;
        int rank = 0;
        for (int q = 0; q < P; ++q) {
            const int eq = __shfl_sync(0xffffffffu, ep, q);
            rank += (eq < ep) || (eq == ep && q < lane);
        }
        if (lane < P) S.sp[rank] = lane;
        __syncwarp();
        const int er = lane < P ? S.sel_e[S.sp[lane]] : -1;
        const int eprev = __shfl_up_sync(0xffffffffu, er, 1);
        const bool start = lane < P && (lane == 0 || eprev != er);
        const uint32_t starts = __ballot_sync(0xffffffffu, start);
        const int d = __popc(starts & ((2u << lane) - 1u)) - 1;
        if (start) {
            S.dex[d] = er;
            S.dstart[d] = lane;
        }
        if (lane < P) S.pdi[S.sp[lane]] = d;
        if (lane == 0) {
            S.nd = __popc(starts);
            S.dstart[__popc(starts)] = P;
        }
        if (blockIdx.x == 0 && lane < P) {
            p.sorted_pair[lane] = S.sp[lane];
            p.pair_row[S.sp[lane]] = lane;
        }
    }
    __syncthreads();
    const int nd = S.nd;
    const unsigned tag = S.tag;
    const int n_gu = nd * p.gu_ntiles;
    const int u0 = S.pf0[nd], u1 = S.pf1[nd];
    const uint32_t dn_unit = (uint32_t)nd * p.dn_tile_bytes;
    if (tracing && tid == 0) trace[9] = globaltimer();

    // ---- 3. one thread issues every weight load of this CTA now -------------------
    if (tid == 0) {
        for (int u = u0; u < u1; ++u) mbar_init(mbar0 + 8 * (u - u0), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        uint32_t off = 0;
        const uint32_t wb = smem_addr(wbuf);
        for (int u = u0; u < u1; ++u) {
            const uint32_t bar = mbar0 + 8 * (u - u0);
            if (u < n_gu) {
                const int dd = u / p.gu_ntiles, tile = u - dd * p.gu_ntiles;
                const size_t tile_id = (size_t)S.dex[dd] * p.gu_ntiles + tile;
                mbar_expect_tx(bar, p.gu_tile_bytes);
                bulk_g2s(wb + off, p.gu_tiles + tile_id * p.gu_tile_bytes, p.gu_tile_bytes, bar);
                off += p.gu_tile_bytes;
            } else {
                const int j = u - n_gu;
                mbar_expect_tx(bar, dn_unit);
                for (int dd = 0; dd < nd; ++dd) {
                    const size_t tile_id = (size_t)S.dex[dd] * (H / 16) + j;
                    bulk_g2s(wb + off + dd * p.dn_tile_bytes, p.dn_tiles + tile_id * p.dn_tile_bytes, p.dn_tile_bytes,
                             bar);
                }
                off += dn_unit;
            }
        }
        if (tracing) trace[1] = globaltimer();
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

    // ---- 4. x as f16x2 with a power-of-two shift per token --------------------------
    for (int t = 0; t < T; ++t) {
        const uint32_t* xrow32 = reinterpret_cast<const uint32_t*>(xr + t * H);
        float m = 0.0f;
        for (int r = tid; r < H / 2; r += kDecThreads) {
            const uint32_t two = xrow32[r];
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
            const uint32_t two = xrow32[r];
            xs[t * xrow + padrow(r)] = f32x2_to_f16x2_rn(bf16_bits_to_f32((uint16_t)(two & 0xffff)) * scl,
                                                        bf16_bits_to_f32((uint16_t)(two >> 16)) * scl);
        }
        __syncthreads();
    }
    if (tracing && tid == 0) trace[2] = globaltimer();

    // ---- 5. gate_up units -> tagged act ------------------------------------------------
    const int c = tid % C, g = tid / C;
    const bool gvalid = g < G;
    uint32_t off = 0;
    int u = u0;
    for (; u < u1 && u < n_gu; ++u) {
        const uint32_t bar = mbar0 + 8 * (u - u0);
        if (!mbar_wait0(bar, p.timeout_ns)) {
            if (tid == 0) { atomicOr(p.status, kDevLoadTimeout); S.abort = 1; }
        }
        __syncthreads();
        if (S.abort) break;
        const int dd = u / p.gu_ntiles, tile = u - dd * p.gu_ntiles;
        const uint8_t* cbase = wbuf + off;
        const uint16_t* sbase = reinterpret_cast<const uint16_t*>(wbuf + off + (H / 2) * TW);
        uint4 q[16];
        float sc[16];
        if (gvalid) {
#pragma unroll
            for (int i = 0; i < 16; ++i) q[i] = *reinterpret_cast<const uint4*>(cbase + (i * G + g) * TW + 16 * c);
            const uint4 s0 = *reinterpret_cast<const uint4*>(sbase + g * TW + 16 * c);
            const uint4 s1 = *reinterpret_cast<const uint4*>(sbase + g * TW + 16 * c + 8);
            const uint32_t sw[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                sc[2 * i] = bf16_bits_to_f32((uint16_t)(sw[i] & 0xffff));
                sc[2 * i + 1] = bf16_bits_to_f32((uint16_t)(sw[i] >> 16));
            }
        }
        for (int r = S.dstart[dd]; r < S.dstart[dd + 1]; ++r) {
            const int pid = S.sp[r], t = pid / k;
            float acc[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) acc[j] = 0.0f;
            if (gvalid) {
                const uint32_t* xrw = xs + t * xrow;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const uint32_t x2 = xrw[padrow(16 * g + i)];
                    const uint32_t words[4] = {q[i].x, q[i].y, q[i].z, q[i].w};
#pragma unroll
                    for (int wd = 0; wd < 4; ++wd) {
                        uint32_t h[4];
                        e2m1x8_to_f16x2x4(words[wd], h);
#pragma unroll
                        for (int b = 0; b < 4; ++b) acc[4 * wd + b] = fma2_f16_f32(h[b], x2, acc[4 * wd + b]);
                    }
                }
#pragma unroll
                for (int j = 0; j < 16; ++j) acc[j] *= sc[j];
            }
            const int col0 = butterfly16<C>(acc, lane);
#pragma unroll
            for (int j = 0; j < Butterfly<C>::NOUT; ++j) red[warp * TW + 16 * c + col0 + j] = acc[j];
            __syncthreads();
            if (tid < TN) {
                float gs = 0.0f, us = 0.0f;
#pragma unroll
                for (int w2 = 0; w2 < kDecWarps; ++w2) {
                    gs += red[w2 * TW + tid];
                    us += red[w2 * TW + TN + tid];
                }
                const float m = pow2f(S.xshift[t]);
                const float a = silu_mul(gs * m, us * m);
                st_volatile_u64(p.act + (size_t)pid * I + tile * TN + tid,
                                ((unsigned long long)tag << 32) | __float_as_uint(a));
            }
            __syncthreads();
        }
        off += p.gu_tile_bytes;
    }
    if (tracing && tid == 0) trace[3] = globaltimer();

    // ---- 6. down units: read act back (tagged), compute, combine ------------------------
    if (u < u1 && !S.abort) {
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
                const unsigned long long t0 = globaltimer();
                bool late = false;
                while (__any_sync(0xffffffffu, pending != 0) && !late) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        if ((pending >> i) & 1u) {
                            ld_volatile_2u64(src + 2 * (lane + 32 * i), a0[i], a1[i]);
                            if ((unsigned)(a0[i] >> 32) == tag && (unsigned)(a1[i] >> 32) == tag) pending &= ~(1u << i);
                        }
                    }
                    late = __any_sync(0xffffffffu, globaltimer() - t0 > p.timeout_ns);
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
                    as[pp * arow + padrow(r)] = f32x2_to_f16x2_rn(__uint_as_float((uint32_t)a0[i]) * scl,
                                                                 __uint_as_float((uint32_t)a1[i]) * scl);
            }
        }
        __syncthreads();
    }
    if (tracing && tid == 0) trace[4] = globaltimer();
    for (; u < u1; ++u) {
        const uint32_t bar = mbar0 + 8 * (u - u0);
        if (!mbar_wait0(bar, p.timeout_ns)) {
            if (tid == 0) { atomicOr(p.status, kDevLoadTimeout); S.abort = 1; }
        }
        __syncthreads();
        const int j = u - n_gu;
        const uint32_t cb = (uint32_t)(I / 2) * 16;
        if (!S.abort) {
            for (int pp = warp; pp < P; pp += kDecWarps) {
                const int di = S.pdi[pp];
                const uint8_t* cbase = wbuf + off + di * p.dn_tile_bytes;
                const uint16_t* sbase = reinterpret_cast<const uint16_t*>(cbase + cb);
                const uint32_t* ar = as + pp * arow;
                float tot[16];
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) tot[jj] = 0.0f;
                if (lane < Gd) {
                    const int gg = lane;
                    float acc[16];
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj) acc[jj] = 0.0f;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const uint4 qq = *reinterpret_cast<const uint4*>(cbase + (i * Gd + gg) * 16);
                        const uint32_t x2 = ar[padrow(16 * gg + i)];
                        const uint32_t words[4] = {qq.x, qq.y, qq.z, qq.w};
#pragma unroll
                        for (int wd = 0; wd < 4; ++wd) {
                            uint32_t h[4];
                            e2m1x8_to_f16x2x4(words[wd], h);
#pragma unroll
                            for (int b = 0; b < 4; ++b) acc[4 * wd + b] = fma2_f16_f32(h[b], x2, acc[4 * wd + b]);
                        }
                    }
                    const uint4 s0 = *reinterpret_cast<const uint4*>(sbase + gg * 16);
                    const uint4 s1 = *reinterpret_cast<const uint4*>(sbase + gg * 16 + 8);
                    const uint32_t sw[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        tot[2 * i] = acc[2 * i] * bf16_bits_to_f32((uint16_t)(sw[i] & 0xffff));
                        tot[2 * i + 1] = acc[2 * i + 1] * bf16_bits_to_f32((uint16_t)(sw[i] >> 16));
                    }
                }
                const int col0 = butterfly16<1>(tot, lane);
                if ((lane & 1) == 0) S.ob[pp * 16 + col0] = tot[0] * pow2f(S.ashift[pp]);
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
    if (tracing && tid == 0) trace[5] = globaltimer();

    // ---- 7. never leave with copies in flight --------------------------------------------
    if (S.abort && tid == 0)
        for (int uu = u0; uu < u1; ++uu) mbar_wait0(mbar0 + 8 * (uu - u0), p.timeout_ns);
}

}  // namespace fe
