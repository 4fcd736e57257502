// Large-T grouped projections on the 5th-generation tensor cores (tcgen05).
//
// "FireEcho Engine", sections "The Goliath Kernel: Why It's Fast" (packed FP4
// bytes are what is read; they are dequantised on chip, next to the tensor
// cores; the expert ids come from device memory) and "Speed Optimization
// History" (grouped dispatch: every routed expert's tokens in one launch).
// With thousands of tokens per layer the projections are dense contractions,
// so here they run as GEMM tiles:
//
//   * A (M = 256 weight columns of one expert, two 128-row accumulators) is
//     built per 64-wide K chunk: the chunk's E2M1 codes and BF16 group scales
//     are staged by cp.async, CUDA cores turn them into f16 values
//     (code value x group scale, exact in f16 when the scale lies in
//     [2^-13, 2^13], which the handle checks once at load time) and write them
//     into the 128-byte-swizzled K-major layout the tensor core reads;
//   * B (N <= 256 token rows of that expert, f16 with a power-of-two shift per
//     row) is gathered by cp.async straight into the same layout;
//   * one thread issues tcgen05.mma kind::f16 into fp32 accumulators in tensor
//     memory (TMEM) and commits each chunk to an mbarrier, so the loads and the
//     dequantisation of later chunks overlap the tensor-core work;
//   * the epilogue reads TMEM with tcgen05.ld: gate_up applies SiLU(gate)*up
//     (gate and up columns sit in adjacent rows) and writes act, down writes
//     o for the ordered combine, both as bf16 (the sums are fp32 until then).
//
// No TMA and no cluster features are used: every load is this CTA's own.
#pragma once

#include "common.cuh"
#include "mma.cuh"

namespace fe {

constexpr int kTcDqWarps = 4;     // warps 0-3: dequantise A
constexpr int kTcLdWarps = 4;     // warps 4-7: cp.async loads
constexpr int kTcMmaWarp = 8;     // warp 8: TMEM allocation and the MMAs
constexpr int kTcThreads = 32 * (kTcDqWarps + kTcLdWarps + 1);
constexpr int kTcDqThreads = 32 * kTcDqWarps, kTcLdThreads = 32 * kTcLdWarps;
constexpr int kTcM = 256;         // A rows (weight columns) per tile: two 128-row accumulators
constexpr int kTcN = 256;         // B rows (tokens) per tile
constexpr int kTcAStages = 3;     // f16 A tiles
constexpr int kTcInStages = 3;    // raw code/scale chunks and f16 B tiles (one index)
constexpr uint32_t kTcABytes = kTcM * 128;            // one f16 A chunk: 256 rows x 64 k
constexpr uint32_t kTcBBytes = kTcN * 128;            // one f16 B chunk: 256 rows x 64 k
constexpr uint32_t kTcRawBytes = 16 * 512 + 16 * 64;  // 16 blocks: one quad of codes + its scales
constexpr uint32_t kTcTmemCols = 512;                 // two 256-column fp32 accumulators
// mbarrier kinds (offsets into the barrier array)
constexpr int kRawFull = 0, kBFull = kTcInStages, kInEmpty = 2 * kTcInStages, kAFull = 3 * kTcInStages,
              kAEmpty = 3 * kTcInStages + kTcAStages, kAccFull = 3 * kTcInStages + 2 * kTcAStages,
              kTcBars = kAccFull + 1;

// Dynamic shared memory: 1024 bytes of alignment slack, then the rings, then
// the barriers and the TMEM address.
__host__ __device__ inline uint32_t tc_smem_bytes()
{
    return 1024 + kTcAStages * kTcABytes + kTcInStages * (kTcBBytes + kTcRawBytes) + 8 * kTcBars + 16 + 4 * kTcN;
}

struct TcParams {
    const uint8_t* blocks;     // gate_up: [E][I/16] units of (gate block, up block); down: [E][H/16] blocks
    int K;                     // reduction length: H (gate_up) or I (down)
    int blocks_per_expert;     // 16-column blocks of one expert: 2 * I/16 (gate_up) or H/16 (down)
    const int32_t* tiles;      // [n][3]: expert, first sorted position, rows (<= kTcN)
    const int32_t* n_tiles;    // [1]
    const uint16_t* bsrc;      // f16 rows: gate_up x [T][H] (row = token), down act [P][I] (row = position)
    const int32_t* bshift;     // power-of-two shift of each B row (token or position)
    const int32_t* sorted_pair;  // gate_up: the token of a sorted position is sorted_pair[pos] / top_k
    int top_k;
    float* out;                // gate_up: act [P][I]; down: o [P][H]; bf16, rows by sorted position
    int out_ld;                // I or H
    uint32_t* status;
    unsigned long long timeout_ns;
    unsigned long long* trace;   // optional: clock64 stamps of tile (0, 0), [3 per chunk]
    unsigned long long* tile_trace;   // optional: [slot][A tile][4] %globaltimer: start, loop end, end, SM
};

// ---- PTX wrappers ------------------------------------------------------------------

// Shared-memory matrix descriptor for a K-major operand in the 128-byte swizzle
// layout: rows of 128 bytes (64 f16), groups of 8 rows 1024 bytes apart.
FE_DEV uint64_t tc_smem_desc(uint32_t saddr)
{
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);   // start address, 16-byte units
    d |= (uint64_t)1u << 16;                            // leading byte offset (not used by this layout)
    d |= (uint64_t)(1024u >> 4) << 32;                  // stride byte offset: 8-row groups
    d |= (uint64_t)1u << 46;                            // descriptor version of tcgen05
    d |= (uint64_t)2u << 61;                            // 128-byte swizzle
    return d;
}

// Instruction descriptor of kind::f16: f32 accumulator, f16 A and B, both K-major.
__host__ __device__ constexpr uint32_t tc_instr_desc(int M, int N)
{
    return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

FE_DEV void tc_mma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accumulate)
{
    const uint32_t mask = 0u;
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(mask), "r"(mask), "r"(mask),
        "r"(mask));
}

FE_DEV void tc_commit(uint32_t mbar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
                 : "memory");
}

FE_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
FE_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

FE_DEV void tc_alloc(uint32_t dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}

FE_DEV void tc_relinquish() { asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory"); }

FE_DEV void tc_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// 16 consecutive fp32 columns of this thread's TMEM lane.
FE_DEV void tc_ld16(uint32_t taddr, uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

FE_DEV void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

FE_DEV void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// 16-byte cp.async; src_bytes 0 fills the destination with zeros.
FE_DEV void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

FE_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

template <int N>
FE_DEV void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

FE_DEV uint32_t tc_saddr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

FE_DEV void tc_mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Bounded wait for the completion of phase `parity` of an mbarrier.  Polls
// with test_wait (no suspension): a thread suspended in try_wait was seen to
// sleep for microseconds past the commit of the MMAs it waited for.
FE_DEV bool tc_mbar_wait(uint32_t bar, uint32_t parity, unsigned long long timeout_ns)
{
    unsigned long long t0 = 0;
    for (int it = 0;; ++it) {
        uint32_t ok;
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

// Byte offset of 16-byte chunk c of row r in a 128-byte-swizzled K-major tile.
FE_DEV uint32_t tc_swz(int r, int c) { return (uint32_t)r * 128u + (uint32_t)((c ^ (r & 7)) << 4); }

// ---- the grouped GEMM tile ---------------------------------------------------------
// grid: (A tiles of one expert, tile slots); block: kTcThreads.  Tile slot y
// holds tiles[y] = (expert e, first sorted position pos0, rows); slots past
// n_tiles exit at once.  Warp roles, linked only by mbarriers in the K loop:
//   warps 0-3  dequantise chunk i's codes into the A ring (stage i % kTcAStages)
//              once its raw bytes have landed and the MMAs of chunk i - 3 are done;
//   warps 4-7  load chunk i's codes, scales and token rows with cp.async into
//              stage i % kTcInStages once the MMAs of chunk i - 3 are done, and
//              let the copies' completion arrive on the stage's "full" barriers;
//   warp 8     issues chunk i's 8 MMAs when its A and B stages are full and
//              commits them to the stages' "empty" barriers.
// After the loop all warps meet, warps 0-7 read the accumulators.
template <bool GATE_UP>
__global__ void __launch_bounds__(kTcThreads, 1) tc_gemm_kernel(TcParams p)
{
    extern __shared__ uint8_t tc_dyn[];
    if ((int)blockIdx.y >= *p.n_tiles) return;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    unsigned long long* ttr = p.tile_trace ? p.tile_trace + 4 * ((size_t)blockIdx.y * gridDim.x + blockIdx.x) : nullptr;
    if (ttr && tid == 0) {
        ttr[0] = globaltimer_ns();
        unsigned smid;
        asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
        ttr[3] = smid;
    }
    const int g = lane >> 2, t = lane & 3;
    const int e = p.tiles[3 * blockIdx.y], pos0 = p.tiles[3 * blockIdx.y + 1], rows = p.tiles[3 * blockIdx.y + 2];
    const int mt = blockIdx.x;
    const int K = p.K, nk = K / 64;
    const int nb = (rows + 15) & ~15;   // MMA N: tile rows rounded up to 16

    // carve the 1024-aligned rings out of the dynamic buffer
    const uint32_t base0 = tc_saddr(tc_dyn);
    const uint32_t pad = (1024u - (base0 & 1023u)) & 1023u;
    uint8_t* sm = tc_dyn + pad;
    uint8_t* a_ring = sm;
    uint8_t* b_ring = a_ring + kTcAStages * kTcABytes;
    uint8_t* raw_ring = b_ring + kTcInStages * kTcBBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(raw_ring + kTcInStages * kTcRawBytes);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kTcBars);
    volatile int* flags = reinterpret_cast<volatile int*>(tmem_slot + 1);                    // [0]: abort
    float* rmul = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(tmem_slot) + 16);     // [kTcN] row scale
    const uint32_t a_addr = tc_saddr(a_ring), b_addr = tc_saddr(b_ring), raw_addr = tc_saddr(raw_ring);
    const uint32_t bar0 = tc_saddr(bars);
    auto bar = [&](int kind, int s) { return bar0 + 8u * (uint32_t)(kind + s); };

    // 2^shift of every B row: undoes the row's power-of-two scaling in the epilogue
    for (int r = tid; r < kTcN; r += kTcThreads) {
        float m = 0.0f;
        if (r < rows) {
            const int pos = pos0 + r;
            m = pow2f(p.bshift[GATE_UP ? p.sorted_pair[pos] / p.top_k : pos]);
        }
        rmul[r] = m;
    }
    if (tid == 0) {
        for (int s = 0; s < kTcInStages; ++s) {
            tc_mbar_init(bar(kRawFull, s), kTcLdThreads);
            tc_mbar_init(bar(kBFull, s), kTcLdThreads);
            tc_mbar_init(bar(kInEmpty, s), 1);
        }
        for (int s = 0; s < kTcAStages; ++s) {
            tc_mbar_init(bar(kAFull, s), kTcDqThreads);
            tc_mbar_init(bar(kAEmpty, s), 1);
        }
        tc_mbar_init(bar(kAccFull, 0), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        flags[0] = 0;
    }
    if (warp == kTcMmaWarp) {
        tc_alloc(tc_saddr(tmem_slot), kTcTmemCols);
        tc_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint8_t* blk0 = p.blocks + ((size_t)e * p.blocks_per_expert + 16 * mt) * (size_t)(9 * K);

    if (warp < kTcDqWarps) {
        // ---- dequantise: raw codes x group scales -> f16 A rows ------------------------
        for (int i = 0; i < nk; ++i) {
            const int si = i % kTcInStages, sa = i % kTcAStages;
            if (!tc_mbar_wait(bar(kRawFull, si), (i / kTcInStages) & 1, p.timeout_ns) ||
                (i >= kTcAStages && !tc_mbar_wait(bar(kAEmpty, sa), ((i - kTcAStages) / kTcAStages) & 1, p.timeout_ns)))
                flags[0] = 1;
            if (flags[0]) break;
            const uint8_t* raw = raw_ring + si * kTcRawBytes;
            uint8_t* A = a_ring + sa * kTcABytes;
#pragma unroll
            for (int m = 0; m < 16 / kTcDqWarps; ++m) {
                const int bi = (16 / kTcDqWarps) * warp + m;
                const uint4 cw = *reinterpret_cast<const uint4*>(raw + bi * 512 + 16 * lane);
                const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
                const uint32_t* sc = reinterpret_cast<const uint32_t*>(raw + 8192 + bi * 64);
                __half2 s2[2][2];
#pragma unroll
                for (int gi = 0; gi < 2; ++gi) {
                    const uint32_t sw = sc[gi * 8 + g];
                    s2[gi][0] = __half2half2(__float2half_rn(bf16_bits_to_f32((uint16_t)(sw & 0xffffu))));
                    s2[gi][1] = __half2half2(__float2half_rn(bf16_bits_to_f32((uint16_t)(sw >> 16))));
                }
#pragma unroll
                for (int s4 = 0; s4 < 4; ++s4) {
                    uint32_t h[4];
                    e2m1x8_to_f16x2x4(words[s4], h);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int col = g + 8 * (j & 1);
                        // gate_up: unit bi/2 owns rows 32 (bi/2) .. +31, gate columns first, up 16 rows
                        // later (row & 7 = col & 7: the 8 lanes of a store hit 8 swizzle phases)
                        const int row = GATE_UP ? 32 * (bi >> 1) + 16 * (bi & 1) + col : 16 * bi + col;
                        const int chunk = 2 * s4 + (j >> 1);
                        __half2 v = *reinterpret_cast<const __half2*>(&h[j]);
                        v = __hmul2(v, s2[s4 >> 1][j & 1]);
                        *reinterpret_cast<__half2*>(A + tc_swz(row, chunk) + 4 * t) = v;
                    }
                }
            }
            fence_proxy_async_smem();
            asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar(kAFull, sa)) : "memory");
        }
    } else if (warp < kTcDqWarps + kTcLdWarps) {
        // ---- load: codes + scales and token rows of chunk i ------------------------------
        const int lt = tid - kTcDqThreads;
        const int c = lt & 7;
        const uint16_t* brow[16];
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            const int r = (lt >> 3) + 16 * m;
            const uint16_t* src = p.bsrc;
            if (r < rows) {
                const int pos = pos0 + r;
                src = p.bsrc + (size_t)(GATE_UP ? p.sorted_pair[pos] / p.top_k : pos) * K;
            }
            brow[m] = src;
        }
        for (int i = 0; i < nk; ++i) {
            const int s = i % kTcInStages;
            if (i >= kTcInStages && !tc_mbar_wait(bar(kInEmpty, s), ((i - kTcInStages) / kTcInStages) & 1, p.timeout_ns))
                flags[0] = 1;
            if (flags[0]) break;
            const uint32_t rdst = raw_addr + s * kTcRawBytes;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int cc = lt + kTcLdThreads * m, bi = cc >> 5, w16 = cc & 31;
                cp_async16(rdst + bi * 512 + 16 * w16, blk0 + (size_t)bi * (9 * K) + 512 * i + 16 * w16, 16);
            }
            if (lt < 64) {
                const int bi = lt >> 2, w16 = lt & 3;
                cp_async16(rdst + 8192 + bi * 64 + 16 * w16, blk0 + (size_t)bi * (9 * K) + 8 * K + 64 * i + 16 * w16, 16);
            }
            asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar(kRawFull, s)) : "memory");
            const uint32_t bdst = b_addr + s * kTcBBytes;
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                const int r = (lt >> 3) + 16 * m;
                cp_async16(bdst + tc_swz(r, c), brow[m] + 64 * i + 8 * c, r < rows ? 16u : 0u);
            }
            asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar(kBFull, s)) : "memory");
        }
        cp_async_wait<0>();   // no copy outlives the loop
    } else {
        // ---- one thread issues the MMAs of every chunk -----------------------------------
        const uint32_t idesc = tc_instr_desc(128, nb);
        int issued = -1;
        for (int i = 0; i < nk; ++i) {
            const int si = i % kTcInStages, sa = i % kTcAStages;
            if (!tc_mbar_wait(bar(kAFull, sa), (i / kTcAStages) & 1, p.timeout_ns) ||
                !tc_mbar_wait(bar(kBFull, si), (i / kTcInStages) & 1, p.timeout_ns))
                flags[0] = 1;
            if (flags[0]) break;
            tc_fence_after();
            if (lane == 0) {
                if (p.trace && blockIdx.x == 0 && blockIdx.y == 0 && i < 64) p.trace[i] = (unsigned long long)clock64();
                const uint32_t aa = a_addr + sa * kTcABytes;
                const uint32_t ba = b_addr + si * kTcBBytes;
#pragma unroll
                for (int acc = 0; acc < 2; ++acc)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        tc_mma_f16(tmem + 256 * acc, tc_smem_desc(aa + acc * (kTcABytes / 2) + 32 * ks),
                                   tc_smem_desc(ba + 32 * ks), idesc, (i > 0 || ks > 0) ? 1u : 0u);
                tc_commit(bar(kAEmpty, sa));
                tc_commit(bar(kInEmpty, si));
            }
            __syncwarp();
            issued = i;
        }
        if (lane == 0 && issued >= 0) tc_commit(bar(kAccFull, 0));   // every MMA issued so far
        __syncwarp();
        // never leave with MMAs in flight (bounded): they read shared memory and TMEM
        if (issued >= 0 && !tc_mbar_wait(bar(kAccFull, 0), 0, p.timeout_ns)) flags[0] = 1;
        if (issued < nk - 1) flags[0] = 1;
    }
    __syncthreads();
    if (ttr && tid == 0) ttr[1] = globaltimer_ns();

    // ---- epilogue: TMEM -> registers -> global ---------------------------------------------
    const bool abort = flags[0] != 0;
    if (abort) {
        if (tid == 0) atomicOr(p.status, kDevTcTimeout);
    } else {
        tc_fence_after();
        // 32 tokens at a time: TMEM -> registers -> a [token][column] tile in the
        // (now idle) A ring -> coalesced 16-byte row stores
        constexpr int OC = GATE_UP ? kTcM / 2 : kTcM;   // output columns of the tile
        const int ocol0 = GATE_UP ? (kTcM / 2) * mt : kTcM * mt;
#pragma unroll 1
        for (int c0 = 0; c0 < nb; c0 += 32) {
            // two staging tiles [32][OC] (column j of token n stored at j ^ (n & 16), so the
            // gate and up lanes of one column, writing tokens n and n + 16, use different banks)
            float* st = reinterpret_cast<float*>(a_ring) + ((c0 >> 5) & 1) * (32 * OC);
            if (warp < 8) {
                // warps 0-3 read accumulator 0, warps 4-7 accumulator 1 (TMEM lanes 32 (warp % 4) ...)
                const int acc = warp >> 2;
                const int row = 128 * acc + 32 * (warp & 3) + lane;   // A row of this thread's TMEM lane
                uint32_t r[32];
                const uint32_t ta = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + 256 * acc + c0;
                tc_ld16(ta, *reinterpret_cast<uint32_t(*)[16]>(&r[0]));
                tc_ld16(ta + 16, *reinterpret_cast<uint32_t(*)[16]>(&r[16]));
                tc_wait_ld();
                if (GATE_UP) {
                    // lanes l and l + 16 hold gate and up of one act column: the gate lane
                    // takes tokens 0-15, the up lane tokens 16-31
                    const bool up = lane & 16;
                    const int acol = 16 * (row >> 5) + (lane & 15);   // act column within the tile
#pragma unroll
                    for (int n = 0; n < 16; ++n) {
                        const float lo = __uint_as_float(r[n]), hi = __uint_as_float(r[16 + n]);
                        const float other = __shfl_xor_sync(0xffffffffu, up ? lo : hi, 16);   // what the partner needs
                        const int tn = up ? 16 + n : n;
                        const float own = up ? hi : lo;
                        const float gv = up ? other : own, uv = up ? own : other;
                        const float m = rmul[c0 + tn];
                        const float gs = gv * m;
                        st[tn * OC + (acol ^ (tn & 16))] = __fdividef(gs, 1.0f + __expf(-gs)) * (uv * m);
                    }
                } else {
#pragma unroll
                    for (int n = 0; n < 32; ++n) st[n * OC + (row ^ (n & 16))] = __uint_as_float(r[n]) * rmul[c0 + n];
                }
            }
            __syncthreads();
            const int nrows = min(32, rows - c0);
            {
                // act (gate_up) and o (down) as bf16, 8 values per 16-byte store: the next
                // kernel (row conversion, ordered combine) reads half the bytes
                constexpr int V8 = OC / 8;
                uint16_t* o16 = reinterpret_cast<uint16_t*>(p.out);
                for (int idx = tid; idx < nrows * V8; idx += kTcThreads) {
                    const int n = idx / V8, v = idx - n * V8;
                    const float4* rowp = reinterpret_cast<const float4*>(st + n * OC);
                    const float4 a = rowp[(2 * v) ^ ((n & 16) >> 2)], b = rowp[(2 * v + 1) ^ ((n & 16) >> 2)];
                    uint4 w;
                    w.x = bf16x2_rn(a.x, a.y);
                    w.y = bf16x2_rn(a.z, a.w);
                    w.z = bf16x2_rn(b.x, b.y);
                    w.w = bf16x2_rn(b.z, b.w);
                    reinterpret_cast<uint4*>(o16 + (size_t)(pos0 + c0 + n) * p.out_ld + ocol0)[v] = w;
                }
            }
            // the next 32 tokens go to the other staging tile: no barrier needed here
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kTcMmaWarp) tc_dealloc(tmem, kTcTmemCols);
    if (ttr && tid == 0) ttr[2] = globaltimer_ns();
}

// ---- small kernels around the tiles -------------------------------------------------

// Tile list: for every expert with tokens, ceil(count / kTcN) tiles of at
// most kTcN sorted positions, experts in ascending order.  One block of 1024
// threads: thread e counts expert e's tiles, a block scan gives its first slot.
__global__ void __launch_bounds__(1024) tc_tiles_kernel(const int32_t* counts, const int32_t* offsets, int E,
                                                        int32_t* tiles, int32_t* n_tiles)
{
    __shared__ int wsum[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int carry = 0;
    for (int e0 = 0; e0 < E; e0 += 1024) {
        const int e = e0 + (int)threadIdx.x;
        const int c = e < E ? counts[e] : 0;
        const int nt = (c + kTcN - 1) / kTcN;
        int incl = nt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            int v = wsum[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += u;
            }
            wsum[lane] = v;   // inclusive over warps
        }
        __syncthreads();
        const int base = carry + (warp > 0 ? wsum[warp - 1] : 0) + incl - nt;
        if (e < E) {
            const int o = offsets[e];
            for (int i = 0; i < nt; ++i) {
                tiles[3 * (base + i)] = e;
                tiles[3 * (base + i) + 1] = o + kTcN * i;
                tiles[3 * (base + i) + 2] = min(kTcN, c - kTcN * i);
            }
        }
        carry += wsum[31];
        __syncthreads();
    }
    if (threadIdx.x == 0) *n_tiles = carry;
}

// Rows of n values -> f16 scaled by 2^-s with s = fp16_shift(row max); one warp
// per row.  BF16: bf16 bits (x, and act as the gate_up tiles leave it); otherwise fp32.
template <bool BF16>
__global__ void tc_rows_to_f16_kernel(const void* src, int rows, int n, uint16_t* dst, int32_t* shift)
{
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    if (warp >= rows) return;
    const size_t base = (size_t)warp * n;
    float m = 0.0f;
    for (int i = lane; i < n / 2; i += 32) {
        float a, b;
        if (BF16) {
            const uint32_t two = static_cast<const uint32_t*>(src)[base / 2 + i];
            a = bf16_bits_to_f32((uint16_t)(two & 0xffffu));
            b = bf16_bits_to_f32((uint16_t)(two >> 16));
        } else {
            const float2 two = static_cast<const float2*>(src)[base / 2 + i];
            a = two.x;
            b = two.y;
        }
        m = fmaxf(m, fmaxf(fabsf(a), fabsf(b)));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const int sh = fp16_shift(m);
    const float sc = pow2f(-sh);
    for (int i = lane; i < n / 2; i += 32) {
        float a, b;
        if (BF16) {
            const uint32_t two = static_cast<const uint32_t*>(src)[base / 2 + i];
            a = bf16_bits_to_f32((uint16_t)(two & 0xffffu));
            b = bf16_bits_to_f32((uint16_t)(two >> 16));
        } else {
            const float2 two = static_cast<const float2*>(src)[base / 2 + i];
            a = two.x;
            b = two.y;
        }
        reinterpret_cast<uint32_t*>(dst)[base / 2 + i] = f32x2_to_f16x2_rn(a * sc, b * sc);
    }
    if (lane == 0) shift[warp] = sh;
}

// Scale check for the tensor-core path: code value x scale is an exact f16
// for every code when each nonzero |scale| lies in [2^-13, 2^13); sets *bad
// otherwise (also for inf / NaN).
__global__ void tc_scale_check_kernel(const uint16_t* scales, size_t n, uint32_t* bad)
{
    uint32_t b = 0;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const uint32_t v = scales[i];
        const uint32_t ex = (v >> 7) & 0xffu;
        b |= ((v & 0x7fffu) != 0u) && (ex < 114u || ex >= 140u);
    }
    if (__any_sync(0xffffffffu, b != 0) && (threadIdx.x & 31) == 0) atomicOr(bad, 1u);
}

}  // namespace fe
