// fe_moe C ABI: handle, workspace, weight loading and the forward enqueue.
// The declarations and the contract of every entry point are in
// include/fe_moe.h.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/fe_moe.h"
#include "common.cuh"
#include "decode.cuh"
#include "gemv.cuh"
#include "gemv_canonical.cuh"
#include "gmma.cuh"
#include "nvfp4.cuh"
#include "pack.cuh"
#include "route.cuh"
#include "route_large.cuh"
#include "router.cuh"
#include "stack_decode.cuh"
#include "stream.cuh"
#include "tcgen05.cuh"

namespace fe_host {
void pack(const float* W, int64_t E, int64_t K, int64_t N, uint8_t* codes, uint16_t* scales);
void pack_int2(const float* W, int64_t E, int64_t K, int64_t N, uint8_t* codes, uint16_t* scales);
}

struct fe_moe_s {
    int E = 0, H = 0, I = 0;
    int device = 0;
    int path = 0;
    int sm_count = 0;
    int smem_optin = 0;
    // fragment-ordered blocks of 16 columns (pack.cuh): gate_up units of a
    // gate block and its up block, down blocks
    uint8_t* gu_blocks = nullptr;   // [E][I/16] x 18H bytes
    uint8_t* dn_blocks = nullptr;   // [E][H/16] x 9I bytes
    uint8_t* dn_rows = nullptr;     // [E][I/32] x 18H bytes: W_dn in row groups (single-launch decode)
    bool loaded = false;
    // experts held as INT2 codes (fe_moe_load_int2): only the single-launch decode path reads them
    bool has_int2 = false;
    uint8_t* fmt = nullptr;         // [E]: 1 = INT2
    uint8_t* gu2_blocks = nullptr;  // [E][I/16] x 10H bytes: INT2 gate_up units
    uint8_t* dn2_rows = nullptr;    // [E][I/32] x 10H bytes: INT2 row groups of W_dn
    // workspace
    int max_T = 0, max_k = 0;
    int32_t* idx = nullptr;
    float* w = nullptr;
    int32_t* counts = nullptr;
    int32_t* offsets = nullptr;
    int32_t* sorted_pair = nullptr;
    int32_t* pair_row = nullptr;
    int32_t* active = nullptr;
    int32_t* n_active = nullptr;
    int32_t* max_count = nullptr;
    float* act = nullptr;
    float* o = nullptr;
    unsigned long long* dec_part = nullptr; // fused decode: [SMs][kDecMaxT][H] tagged per-CTA partial outputs
    unsigned long long* dec_epoch = nullptr;  // fused decode: per-CTA launch counts, then the arrival counter
    uint32_t dec_plan[fe::kDecMaxT + 1][fe::kDecMaxPairs + 1] = {};   // weight bytes per (T, k); 0: not fused
    bool dec_planned[fe::kDecMaxT + 1][fe::kDecMaxPairs + 1] = {};
    int32_t* sg_table = nullptr;            // streaming kernels: [2][SMs][4] work split
    unsigned long long* trace = nullptr;    // optional phase stamps (caller's buffer)
    // tensor-core path (tcgen05.cuh)
    bool tc_scales_ok = false;              // every group scale in the exact-f16 range
    uint16_t* tc_x = nullptr;               // x rows as f16 [max_T][H]
    int32_t* tc_xshift = nullptr;           // [max_T]
    uint16_t* tc_act = nullptr;             // act rows as f16 [P][I], by sorted position
    int32_t* tc_ashift = nullptr;           // [P]
    int32_t* tc_tiles = nullptr;            // [max tiles][3]
    int32_t* tc_ntiles = nullptr;           // [1]
    int32_t* grp_bh = nullptr;              // grouping for many tokens: [P / kGroupChunk + 1][E]
    // block-scaled FP4 variant (nvfp4.cuh, fe_moe_load_nvfp4): weight tile images and
    // row scales, built at load; token tile images per forward (workspace)
    uint8_t* nv_gu = nullptr;               // [E][2I/128][H/256] x kNvAChunk bytes
    uint8_t* nv_dn = nullptr;               // [E][H/128][I/256] x kNvAChunk bytes
    float* nv_gug = nullptr;                // [E][2I]
    float* nv_dng = nullptr;                // [E][H]
    uint8_t* nv_b = nullptr;                // [tile slots][max(H, I)/256] x kNvBChunk bytes
    float* nv_bg = nullptr;                 // [tile slots][256]
    uint8_t* nv_xc = nullptr;               // x encoded per token: codes [max_T][H/2]
    uint8_t* nv_xs = nullptr;               // scale factors [max_T][H/16]
    float* nv_xg = nullptr;                 // row scales [max_T]
    float* rt_part = nullptr;               // router GEMM: K-split partials (router.cuh)
    unsigned* rt_ticket = nullptr;          // router GEMM: per 16-token tile, CTAs done
    uint32_t* status = nullptr;
    uint16_t* x_stage = nullptr;
    float* logits_stage = nullptr;
    uint16_t* y_stage = nullptr;
    size_t weight_bytes = 0, work_bytes = 0;
    int last_T = 0, last_k = 0;
    int last_path = 0, last_kernels = 0;
    int test_extra_arrivals = 0;            // fe_moe_set_exchange_test
    unsigned long long exchange_timeout_ns = 200ull * 1000 * 1000;
};

struct fe_moe_stack_s {
    std::vector<fe_moe_s*> layers;
    int device = 0, E = 0, H = 0, max_T = 0;
    uint16_t* a_stage = nullptr;     // fe_moe_stack_forward_host: [n + 1][max_T][H] (inputs; chained: all)
    uint16_t* b_stage = nullptr;     // [n][max_T][H] (outputs of independent layers)
    float* logits_stage = nullptr;   // [n][max_T][E]
    bool prefetch = true;            // one persistent launch streams the layers' weights back to back
    // persistent launch (stack_decode.cuh): layer table, tagged partial outputs, counters
    bool persistent_ok = false;      // shapes, sizes and occupancy allow it
    uint32_t stk_smem = 0;
    fe::StackLayer* d_layers = nullptr;        // [n] on the device
    std::vector<fe::StackLayer> h_layers;      // the same on the host: the handles' buffers at creation
    unsigned long long* part = nullptr;        // [3][SMs][H]
    unsigned long long* ctr = nullptr;         // [SMs + 2 kStkBufs]
    int sm_count = 0;
    int last_launches = 0;
};

namespace {

// Text of the last CUDA failure seen by this thread (fe_moe_last_error).
thread_local char g_last_error[256] = "";

fe_status record_cuda(cudaError_t e, const char* where)
{
    snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%d)", where, cudaGetErrorString(e), (int)e);
    return e == cudaErrorMemoryAllocation ? FE_ERR_OOM : FE_ERR_CUDA;
}

#define FE_CUDA_TRY(expr)                                 \
    do {                                                  \
        cudaError_t err__ = (expr);                       \
        if (err__ != cudaSuccess) return record_cuda(err__, #expr); \
    } while (0)

struct DeviceGuard {
    int prev = -1;
    bool ok = true;
    explicit DeviceGuard(int dev)
    {
        if (cudaGetDevice(&prev) != cudaSuccess) { ok = false; return; }
        if (prev != dev && cudaSetDevice(dev) != cudaSuccess) ok = false;
    }
    ~DeviceGuard()
    {
        if (prev >= 0) cudaSetDevice(prev);
    }
};

template <typename T>
cudaError_t dmalloc(T** p, size_t n, size_t* acc)
{
    *p = nullptr;
    if (n == 0) n = 1;
    cudaError_t e = cudaMalloc(reinterpret_cast<void**>(p), n * sizeof(T));
    if (e == cudaSuccess && acc) *acc += n * sizeof(T);
    return e;
}

void free_workspace(fe_moe_s* h)
{
    void* ptrs[] = {h->idx, h->w, h->counts, h->offsets, h->sorted_pair, h->pair_row, h->active, h->n_active,
                    h->max_count, h->act, h->o, h->status, h->x_stage, h->logits_stage, h->y_stage,
                    h->dec_part, h->dec_epoch, h->sg_table, h->tc_x, h->tc_xshift, h->tc_act, h->tc_ashift,
                    h->tc_tiles, h->tc_ntiles, h->grp_bh, h->rt_part, h->rt_ticket, h->nv_b, h->nv_bg,
                    h->nv_xc, h->nv_xs, h->nv_xg};
    for (void* p : ptrs)
        if (p) cudaFree(p);
    h->idx = nullptr; h->w = nullptr; h->counts = nullptr; h->offsets = nullptr; h->sorted_pair = nullptr;
    h->pair_row = nullptr; h->active = nullptr; h->n_active = nullptr; h->max_count = nullptr; h->act = nullptr;
    h->o = nullptr; h->status = nullptr; h->x_stage = nullptr; h->logits_stage = nullptr; h->y_stage = nullptr;
    h->dec_part = nullptr;
    h->dec_epoch = nullptr;
    h->sg_table = nullptr;
    h->tc_x = nullptr; h->tc_xshift = nullptr; h->tc_act = nullptr; h->tc_ashift = nullptr;
    h->tc_tiles = nullptr; h->tc_ntiles = nullptr;
    h->grp_bh = nullptr;
    h->rt_part = nullptr;
    h->rt_ticket = nullptr;
    h->nv_b = nullptr;
    h->nv_bg = nullptr;
    h->nv_xc = h->nv_xs = nullptr;
    h->nv_xg = nullptr;
    h->max_T = h->max_k = 0;
    h->work_bytes = 0;
}

// Tile width TW = 16 * C columns for a matrix with K rows of reduction and N
// columns: one thread per (16-column chunk, 32-k group), at most 256 threads
// per CTA, C a power of two up to 32 dividing the columns (for the fused
// gate_up matrix the tile holds TW/2 gate and TW/2 up columns, so TW/2 must
// divide I).  Returns 0 if no width fits.
int pick_tile_width(int K, int cols, bool gate_up)
{
    const int G = K / 32;
    for (int C = 32; C >= (gate_up ? 2 : 1); C >>= 1) {   // gate_up: 16-byte chunks never straddle gate and up
        if (C * G > 256) continue;
        if (gate_up ? (cols % (8 * C) == 0) : (cols % (16 * C) == 0)) return 16 * C;
    }
    return 0;
}

int roundup32(int v) { return (v + 31) / 32 * 32; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shared-memory bytes the fused decode kernel reserves for weights at (T, k),
// or 0 if the call is outside what it takes: T <= 8 tokens, T*k <= 16 pairs,
// E <= 512, H <= 2048, at most kDecMaxUnits units per CTA for any number of
// distinct routed experts, the whole plan within the device's shared memory,
// and the kernel resident on every SM at once (its CTAs wait for each other).
// Computed once per (T, k) and kept in the handle.
uint32_t decode_weight_bytes(fe_moe_s* h, int T, int k)
{
    if (T < 1 || T > fe::kDecMaxT || k < 1 || k > fe::kDecMaxPairs || T * k > fe::kDecMaxPairs) return 0;
    if (h->dec_planned[T][k]) return h->dec_plan[T][k];
    uint32_t wb = 0;
    const int nd_max = std::min(h->E, T * k);
    const int U = fe::dec_units(nd_max, h->I);
    const int units = (U + h->sm_count - 1) / h->sm_count;
    if (h->E <= fe::kDecMaxE && h->H <= fe::kDecMaxH && h->I <= 1024 && h->sm_count > 0 &&
        h->sm_count <= fe::kDecMaxCtas && units <= fe::kDecMaxUnits &&
        h->dec_part != nullptr) {
        const uint32_t w = ((uint32_t)units * fe::dec_unit_bytes(h->H) + 127u) / 128u * 128u;
        const size_t total = fe::decode_smem_layout(w, T, h->H).total;
        int per_sm = 0;
        if (total <= (size_t)h->smem_optin &&
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fe::decode_kernel, fe::kDecThreads, total) ==
                cudaSuccess &&
            per_sm >= 1)
            wb = w;
    }
    h->dec_plan[T][k] = wb;
    h->dec_planned[T][k] = true;
    return wb;
}

fe_status decode_path(fe_moe_s* h, const void* x, const float* logits, int T, int k, void* y, uint32_t wbytes,
                      cudaStream_t s)
{
    fe::DecodeParams dp{};
    dp.x = static_cast<const uint16_t*>(x);
    dp.logits = logits;
    dp.y = static_cast<uint16_t*>(y);
    dp.T = T; dp.E = h->E; dp.H = h->H; dp.I = h->I; dp.k = k;
    dp.gu_blocks = h->gu_blocks; dp.dn_rows = h->dn_rows;
    dp.fmt = h->has_int2 ? h->fmt : nullptr;
    dp.gu2_blocks = h->gu2_blocks; dp.dn2_rows = h->dn2_rows;
    dp.idx = h->idx; dp.w = h->w; dp.counts = h->counts; dp.offsets = h->offsets;
    dp.sorted_pair = h->sorted_pair; dp.pair_row = h->pair_row;
    dp.part = h->dec_part;
    dp.epoch = h->dec_epoch;
    dp.trace = h->trace;
    dp.status = h->status;
    dp.timeout_ns = 200ull * 1000 * 1000;
    dp.exchange_timeout_ns = h->exchange_timeout_ns;
    dp.extra_arrivals = h->test_extra_arrivals;
    dp.weight_bytes = wbytes;
    dp.bulk_inputs = aligned16(x);   // 2*T*H bytes: a multiple of 16 (H % 64 == 0)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(h->sm_count);
    cfg.blockDim = dim3(fe::kDecThreads);
    cfg.dynamicSmemBytes = fe::decode_smem_layout(wbytes, T, h->H).total;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    FE_CUDA_TRY(cudaLaunchKernelEx(&cfg, fe::decode_kernel, dp));
    return FE_OK;
}

// Opt the kernels into the device's largest dynamic shared memory (once,
// outside any stream capture).  Function attributes are process-wide, so a
// handle of another shape must never lower the limit below what this
// handle's launches request.
// Shapes the tensor-core tiles cover: 128 act columns (64 gate + 64 up pairs of
// rows) and 256 output columns per tile.
bool tc_shape_ok(const fe_moe_s* h) { return h->I % 128 == 0 && h->H % 256 == 0; }

// Shapes of the block-scaled FP4 variant: K stages of 256 for both projections
// (so also 128-row weight tiles of 2I and H).
bool nv_shape_ok(const fe_moe_s* h) { return h->I % 256 == 0 && h->H % 256 == 0; }

// Token-expert pairs from which the automatic path choice takes the tensor
// cores (below it the grouped mma.sync kernels keep the weights' single pass).
constexpr int kTcAutoPairs = 4096;

// Tokens from which routing and grouping run on the whole GPU.
constexpr int kRouteLargeTokens = 32;

size_t tc_max_tiles(const fe_moe_s* h, size_t P)
{
    return (P + fe::kTcN - 1) / fe::kTcN + std::min((size_t)h->E, P);
}

// Streaming kernels: 8-token blocks staged at once (gate_up rows are 4 times
// the bytes of down rows at the 30B-like shape).
constexpr int kSgGateUpBlocks = 2;
constexpr int kSgDownBlocks = 8;
constexpr int kSgStaticReserve = 256;   // static shared bytes of the streaming kernels, rounded up

struct SgPlan {
    int slots = 0, chunk = 0;
    size_t smem = 0;
};

// Largest token chunk (down to 8) that leaves room for min_slots ring slots,
// then as many slots as fit (at most kSgMaxSlots); slots = 0 if nothing fits.
SgPlan sg_plan(const fe_moe_s* h, bool gate_up, int K, uint32_t unit_bytes, int max_blocks, int min_slots, int slot_step)
{
    const size_t limit = (size_t)h->smem_optin - kSgStaticReserve;
    SgPlan best;
    for (int want = min_slots; want >= 2 && best.slots == 0; want = want > 2 ? want - 1 : 1) {
        for (int chunk = 8 * max_blocks; chunk >= 8; chunk -= 8) {
            int slots = 0;
            for (int r = fe::kSgMaxSlots / slot_step * slot_step; r >= want; r -= slot_step)
                if (fe::sg_smem_layout(gate_up, K, unit_bytes, r, chunk).total <= limit) {
                    slots = r;
                    break;
                }
            if (slots) {
                best.slots = slots;
                best.chunk = chunk;
                best.smem = fe::sg_smem_layout(gate_up, K, unit_bytes, slots, chunk).total;
                break;
            }
        }
    }
    return best;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

cudaError_t configure_kernels(const fe_moe_s* h)
{
    const int optin = h->smem_optin;
    cudaError_t e = cudaFuncSetAttribute(fe::route_group_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(fe::gmma_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(fe::gmma_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(fe::decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(fe::tc_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(fe::tc_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(fe::nvfp4_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(fe::nvfp4_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
    // (the streaming kernels hold a little static shared state besides)
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(fe::sg_kernel<true, kSgGateUpBlocks>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 optin - kSgStaticReserve);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(fe::sg_kernel<false, kSgDownBlocks>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 optin - kSgStaticReserve);
    return e;
}

fe_status gemv_path(fe_moe_s* h, const uint16_t* x, int T, int k, cudaStream_t s)
{
    const int P = T * k;
    const int max_active = std::min(h->E, P);
    fe::GmmaParams gp{};
    gp.offsets = h->offsets;
    gp.active = h->active;
    gp.n_active = h->n_active;
    gp.sorted_pair = h->sorted_pair;
    gp.top_k = k;
    gp.status = h->status;
    gp.timeout_ns = 200ull * 1000 * 1000;
    // gate_up + SwiGLU: K = H, units of 16 gate + 16 up columns
    gp.blocks = h->gu_blocks;
    gp.K = h->H;
    gp.n_units = h->I / 16;
    gp.N_out = h->I;
    gp.x = x;
    gp.act_in = nullptr;
    gp.out = h->act;
    fe::gmma_kernel<true><<<max_active * gp.n_units, fe::kGmmaThreads, fe::gmma_smem_bytes(true, h->H), s>>>(gp);
    FE_CUDA_TRY(cudaGetLastError());
    // down: K = I, units of 16 output columns
    gp.blocks = h->dn_blocks;
    gp.K = h->I;
    gp.n_units = h->H / 16;
    gp.N_out = h->H;
    gp.x = nullptr;
    gp.act_in = h->act;
    gp.out = h->o;
    fe::gmma_kernel<false><<<max_active * gp.n_units, fe::kGmmaThreads, fe::gmma_smem_bytes(false, h->I), s>>>(gp);
    FE_CUDA_TRY(cudaGetLastError());
    return FE_OK;
}

// Plans of the two streaming kernels and the work-split arguments the grouping
// step uses to fill the range table; false when a ring does not fit.
struct SgSetup {
    SgPlan gu, dn;
    fe::SgSplit split{};
};

bool stream_setup(const fe_moe_s* h, int T, SgSetup& st)
{
    const uint32_t gu_unit = 2u * fe::block_bytes(h->H), dn_unit = fe::block_bytes(h->I);
    // an expert has at most T pairs: no chunk longer than that
    const int tb = (T + 7) / 8;
    st.gu = sg_plan(h, true, h->H, gu_unit, std::min(kSgGateUpBlocks, tb), 3, 1);
    st.dn = sg_plan(h, false, h->I, dn_unit, std::min(kSgDownBlocks, tb), 16, 1);
    if (st.gu.slots == 0 || st.dn.slots < fe::kSgComputeWarps) return false;
    fe::SgSplit& sp = st.split;
    sp.table = h->sg_table;
    sp.G = h->sm_count;
    // cost of a unit in ~100-cycle units: its bytes at the per-SM share of HBM,
    // the A conversion per chunk, the MMAs per 8-token block, the restaging of
    // a chunk's rows
    const int K[2] = {h->H, h->I};
    const SgPlan* pl[2] = {&st.gu, &st.dn};
    const uint32_t ub[2] = {gu_unit, dn_unit};
    sp.n_units[0] = h->I / 16;
    sp.n_units[1] = h->H / 16;
    for (int ph = 0; ph < 2; ++ph) {
        sp.chunk[ph] = pl[ph]->chunk;
        sp.c_bytes[ph] = std::max(1, (int)(ub[ph] / 2300));
        sp.c_chunk[ph] = std::max(1, K[ph] / 320);
        sp.c_block[ph] = std::max(1, K[ph] / 340);
        sp.c_restage[ph] = std::max(1, (int)((size_t)pl[ph]->chunk * K[ph] * 2 / 6400));
    }
    return true;
}

// Moderate-T path on the streaming kernels: gate_up units (x rows staged as
// fp16 in the kernel, SwiGLU into act), then down units (act rows likewise,
// into o), each CTA on the range the grouping step put in the table.  The
// routing and grouping ran before; the ordered combine runs after.
fe_status stream_path(fe_moe_s* h, const uint16_t* x, int k, const SgSetup& st, cudaStream_t s)
{
    fe::SgParams sp{};
    sp.offsets = h->offsets;
    sp.active = h->active;
    sp.n_active = h->n_active;
    sp.sorted_pair = h->sorted_pair;
    sp.top_k = k;
    sp.status = h->status;
    sp.timeout_ns = 200ull * 1000 * 1000;
    sp.trace = h->trace;
    // gate_up: K = H, units of 16 gate + 16 up columns
    sp.blocks = h->gu_blocks;
    sp.K = h->H;
    sp.n_units = h->I / 16;
    sp.unit_bytes = 2u * fe::block_bytes(h->H);
    sp.N_out = h->I;
    sp.bsrc = x;
    sp.out = h->act;
    sp.slots = st.gu.slots;
    sp.chunk = st.gu.chunk;
    sp.range = h->sg_table;
    FE_CUDA_TRY(launch_pdl(fe::sg_kernel<true, kSgGateUpBlocks>, dim3(h->sm_count), dim3(fe::kSgThreads), st.gu.smem, s, sp));
    // down: K = I, units of 16 output columns, one warp each
    sp.blocks = h->dn_blocks;
    sp.K = h->I;
    sp.n_units = h->H / 16;
    sp.unit_bytes = fe::block_bytes(h->I);
    sp.N_out = h->H;
    sp.bsrc = h->act;
    sp.out = h->o;
    sp.slots = st.dn.slots;
    sp.chunk = st.dn.chunk;
    sp.range = h->sg_table + 4 * (size_t)h->sm_count;
    sp.trace = h->trace ? h->trace + 8 * (size_t)h->sm_count : nullptr;
    FE_CUDA_TRY(launch_pdl(fe::sg_kernel<false, kSgDownBlocks>, dim3(h->sm_count), dim3(fe::kSgThreads), st.dn.smem, s, sp));
    return FE_OK;
}

// Router + grouping outputs (idx, w, counts, offsets, sorted_pair, pair_row,
// active, n_active, max_count) for the non-fused paths: the single-CTA kernel
// for a few tokens, the GPU-wide kernels for many.
fe_status route_and_group(fe_moe_s* h, const float* logits, int T, int k, const fe::SgSplit* split, cudaStream_t s)
{
    const int P = T * k;
    fe::RouteParams rp{};
    rp.logits = logits; rp.T = T; rp.E = h->E; rp.k = k;
    rp.idx = h->idx; rp.w = h->w; rp.counts = h->counts; rp.offsets = h->offsets;
    rp.sorted_pair = h->sorted_pair; rp.pair_row = h->pair_row; rp.active = h->active;
    rp.n_active = h->n_active; rp.max_count = h->max_count; rp.status = h->status;
    if (split) rp.split = *split;
    if (T >= kRouteLargeTokens && fe::route_large_ok(h->E, k)) {
        const int nblk = (P + fe::kGroupChunk - 1) / fe::kGroupChunk;
        fe::route_tokens_kernel<<<(T + fe::kRouteWarps - 1) / fe::kRouteWarps, fe::kRouteWarps * 32, 0, s>>>(rp);
        fe::group_hist_kernel<<<nblk, fe::kGroupThreads, sizeof(int32_t) * h->E, s>>>(h->idx, P, h->E, h->grp_bh);
        const size_t scan_smem = sizeof(int32_t) * 2 * (size_t)((h->E + 1) & ~1) + sizeof(long long) * (2 * ((size_t)h->E + 1) + 32);
        fe::group_scan_kernel<<<1, 1024, scan_smem, s>>>(h->grp_bh, nblk, h->E, h->counts,
                                                                          h->offsets, h->active, h->n_active,
                                                                          h->max_count, rp.split);
        fe::group_scatter_kernel<<<nblk, fe::kGroupThreads, sizeof(int32_t) * h->E * (fe::kGroupThreads / 32 + 1),
                                   s>>>(h->idx, P, h->E, h->grp_bh, h->sorted_pair, h->pair_row, h->status);
    } else {
        const int rthreads = std::min(fe::kRouteMaxThreads, std::max(32, roundup32(std::max(P, 32 * T))));
        fe::route_group_kernel<<<1, rthreads, fe::route_smem_bytes(h->E, rthreads), s>>>(rp);
    }
    FE_CUDA_TRY(cudaGetLastError());
    return FE_OK;
}

// Large-T path on the tensor cores: tile list, x rows to f16, gate_up tiles
// (SwiGLU into act), act rows to f16, down tiles (into o).  The routing and
// grouping ran before; the ordered combine runs after.
fe_status tcgen05_path(fe_moe_s* h, const uint16_t* x, int T, int k, cudaStream_t s)
{
    const int P = T * k;
    const int max_tiles = (int)tc_max_tiles(h, (size_t)P);
    fe::tc_tiles_kernel<<<1, 1024, 0, s>>>(h->counts, h->offsets, h->E, h->tc_tiles, h->tc_ntiles);
    fe::tc_rows_to_f16_kernel<true><<<(T + 7) / 8, 256, 0, s>>>(x, T, h->H, h->tc_x, h->tc_xshift);
    fe::TcParams tp{};
    tp.tiles = h->tc_tiles;
    tp.n_tiles = h->tc_ntiles;
    tp.sorted_pair = h->sorted_pair;
    tp.top_k = k;
    tp.status = h->status;
    tp.timeout_ns = 200ull * 1000 * 1000;
    tp.trace = h->trace;
    tp.tile_trace = h->trace ? h->trace + 1024 : nullptr;
    tp.blocks = h->gu_blocks;
    tp.K = h->H;
    tp.blocks_per_expert = 2 * (h->I / 16);
    tp.bsrc = h->tc_x;
    tp.bshift = h->tc_xshift;
    tp.out = h->act;
    tp.out_ld = h->I;
    fe::tc_gemm_kernel<true><<<dim3(h->I / 128, max_tiles), fe::kTcThreads, fe::tc_smem_bytes(), s>>>(tp);
    FE_CUDA_TRY(cudaGetLastError());
    // act was left as bf16 by the gate_up tiles
    fe::tc_rows_to_f16_kernel<true><<<(P + 7) / 8, 256, 0, s>>>(h->act, P, h->I, h->tc_act, h->tc_ashift);
    tp.blocks = h->dn_blocks;
    tp.K = h->I;
    tp.blocks_per_expert = h->H / 16;
    tp.bsrc = h->tc_act;
    tp.bshift = h->tc_ashift;
    tp.out = h->o;
    tp.out_ld = h->H;
    tp.trace = h->trace ? h->trace + 256 : nullptr;
    tp.tile_trace = h->trace ? h->trace + 1024 + 4 * (size_t)(h->I / 128) * max_tiles : nullptr;
    fe::tc_gemm_kernel<false><<<dim3(h->H / fe::kTcM, max_tiles), fe::kTcThreads, fe::tc_smem_bytes(), s>>>(tp);
    FE_CUDA_TRY(cudaGetLastError());
    return FE_OK;
}

// Token tile images of the block-scaled FP4 variant: slots x K stages.
size_t nv_token_bytes(const fe_moe_s* h, size_t slots)
{
    return slots * (size_t)(std::max(h->H, h->I) / fe::kNvKc) * fe::kNvBChunk;
}

// Workspace of the block-scaled FP4 variant for max_T tokens and P pairs:
// token images of every tile slot, and x encoded per token.
cudaError_t nv_alloc_workspace(fe_moe_s* h, int max_T, size_t P, size_t* acc)
{
    const size_t slots = tc_max_tiles(h, P);
    cudaError_t e = dmalloc(&h->nv_b, nv_token_bytes(h, slots), acc);
    if (e == cudaSuccess) e = dmalloc(&h->nv_bg, slots * fe::kNvN, acc);
    if (e == cudaSuccess) e = dmalloc(&h->nv_xc, (size_t)max_T * (h->H / 2), acc);
    if (e == cudaSuccess) e = dmalloc(&h->nv_xs, (size_t)max_T * (h->H / 16), acc);
    if (e == cudaSuccess) e = dmalloc(&h->nv_xg, (size_t)max_T, acc);
    return e;
}

// Block-scaled FP4 variant (nvfp4.cuh): tile list, x rows gathered into NVFP4
// token images, gate_up tiles (SwiGLU into act, bf16), act rows into token
// images, down tiles (into o, bf16).  Routing and grouping ran before; the
// ordered combine runs after.
fe_status nvfp4_path(fe_moe_s* h, const uint16_t* x, int T, int k, cudaStream_t s)
{
    const int P = T * k;
    const int max_tiles = (int)tc_max_tiles(h, (size_t)P);
    fe::tc_tiles_kernel<<<1, 1024, 0, s>>>(h->counts, h->offsets, h->E, h->tc_tiles, h->tc_ntiles);
    // x encoded once per token, then gathered into the tiles' images
    fe::nvfp4_rows_kernel<true><<<(unsigned)((T + 7) / 8), 256, 0, s>>>(x, T, h->H, h->nv_xc, h->nv_xs, h->nv_xg);
    const unsigned row_blocks = (unsigned)(((size_t)max_tiles * fe::kNvN + 7) / 8);
    fe::nvfp4_gather_rows_kernel<<<row_blocks, 256, 0, s>>>(h->nv_xc, h->nv_xs, h->nv_xg, h->H, h->tc_tiles,
                                                            h->tc_ntiles, h->sorted_pair, k, h->nv_b, h->nv_bg);
    fe::NvParams np{};
    np.tiles = h->tc_tiles;
    np.n_tiles = h->tc_ntiles;
    np.status = h->status;
    np.timeout_ns = 200ull * 1000 * 1000;
    np.b_img = h->nv_b;
    np.b_g = h->nv_bg;
    np.a_img = h->nv_gu;
    np.a_g = h->nv_gug;
    np.MT = 2 * h->I / fe::kNvM;
    np.KC = h->H / fe::kNvKc;
    np.out = reinterpret_cast<uint16_t*>(h->act);
    np.out_ld = h->I;
    fe::nvfp4_gemm_kernel<true><<<dim3(np.MT, max_tiles), fe::kNvThreads, fe::nv_smem_bytes(), s>>>(np);
    FE_CUDA_TRY(cudaGetLastError());
    // act was left as bf16 rows by sorted position
    fe::nvfp4_token_rows_kernel<<<row_blocks, 256, 0, s>>>(reinterpret_cast<const uint16_t*>(h->act), h->I,
                                                           h->tc_tiles, h->tc_ntiles, h->nv_b, h->nv_bg);
    np.a_img = h->nv_dn;
    np.a_g = h->nv_dng;
    np.MT = h->H / fe::kNvM;
    np.KC = h->I / fe::kNvKc;
    np.out = reinterpret_cast<uint16_t*>(h->o);
    np.out_ld = h->H;
    fe::nvfp4_gemm_kernel<false><<<dim3(np.MT, max_tiles), fe::kNvThreads, fe::nv_smem_bytes(), s>>>(np);
    FE_CUDA_TRY(cudaGetLastError());
    return FE_OK;
}

}  // namespace

extern "C" {

const char* fe_moe_status_string(fe_status s)
{
    switch (s) {
        case FE_OK: return "ok";
        case FE_ERR_INVALID_ARG: return "invalid argument";
        case FE_ERR_UNSUPPORTED: return "unsupported";
        case FE_ERR_NOT_LOADED: return "weights not loaded";
        case FE_ERR_CAPACITY: return "T or top_k above the reserved workspace";
        case FE_ERR_OOM: return "device out of memory";
        case FE_ERR_CUDA: return "CUDA error";
        case FE_ERR_DEVICE_STATUS: return "a kernel flagged bad data";
    }
    return "unknown status";
}

fe_status fe_moe_create(int E, int H, int I, int group, fe_moe_t* out)
{
    if (!out) return FE_ERR_INVALID_ARG;
    *out = nullptr;
    if (group != 32) return FE_ERR_UNSUPPORTED;
    if (E < 1 || E > 1024 || H <= 0 || I <= 0 || H % 32 || I % 32) return FE_ERR_INVALID_ARG;
    // gate_up tiles: TW/2 gate + TW/2 up columns, so TW/2 must divide I
    // fragment-ordered blocks: 64-k quads along K, 16-column blocks along N
    if (H % 64 || I % 64) return FE_ERR_UNSUPPORTED;
    if (fe::gmma_smem_bytes(true, H) > 227 * 1024 || fe::gmma_smem_bytes(false, I) > 227 * 1024) return FE_ERR_UNSUPPORTED;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FE_ERR_CUDA;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return FE_ERR_CUDA;
    if (prop.major != 10) return FE_ERR_UNSUPPORTED;
    int optin = 0;
    if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return FE_ERR_CUDA;
    fe_moe_s* h = new (std::nothrow) fe_moe_s();
    if (!h) return FE_ERR_OOM;
    h->E = E; h->H = H; h->I = I; h->device = dev;
    h->sm_count = prop.multiProcessorCount;
    h->smem_optin = optin;
    size_t acc = 0;
    cudaError_t e = cudaSuccess;
    // codes (K/2 bytes per column) + scales (K/32 bf16 per column), same bytes as the packed format
    if (e == cudaSuccess) e = dmalloc(&h->gu_blocks, (size_t)E * (I / 16) * 2 * fe::block_bytes(H), &acc);
    if (e == cudaSuccess) e = dmalloc(&h->dn_blocks, (size_t)E * (H / 16) * fe::block_bytes(I), &acc);
    if (e == cudaSuccess) e = dmalloc(&h->dn_rows, (size_t)E * (I / 32) * 18 * (size_t)H, &acc);
    if (e == cudaSuccess) e = dmalloc(&h->status, 1, &acc);
    if (e == cudaSuccess) e = cudaMemset(h->status, 0, sizeof(uint32_t));
    if (e != cudaSuccess) {
        fe_moe_destroy(h);
        return e == cudaErrorMemoryAllocation ? FE_ERR_OOM : FE_ERR_CUDA;
    }
    h->weight_bytes = acc;
    *out = h;
    return FE_OK;
}

fe_status fe_moe_reserve(fe_moe_t h, int max_T, int max_top_k)
{
    if (!h || max_T < 1 || max_top_k < 1 || max_top_k > h->E) return FE_ERR_INVALID_ARG;
    if ((int64_t)max_T * max_top_k > (int64_t)1 << 26) return FE_ERR_UNSUPPORTED;
    DeviceGuard g(h->device);
    if (!g.ok) return FE_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return FE_ERR_CUDA;
    uint32_t* keep_status = h->status;
    h->status = nullptr;
    free_workspace(h);
    h->status = keep_status;
    const size_t P = (size_t)max_T * max_top_k;
    size_t acc = 0;
    cudaError_t e = cudaSuccess;
    if (e == cudaSuccess) e = dmalloc(&h->idx, P, &acc);
    if (e == cudaSuccess) e = dmalloc(&h->w, P, &acc);
    if (e == cudaSuccess) e = dmalloc(&h->counts, (size_t)h->E, &acc);
    if (e == cudaSuccess) e = dmalloc(&h->offsets, (size_t)h->E + 1, &acc);
    if (e == cudaSuccess) e = dmalloc(&h->sorted_pair, P, &acc);
    if (e == cudaSuccess) e = dmalloc(&h->pair_row, P, &acc);
    if (e == cudaSuccess) e = dmalloc(&h->active, (size_t)h->E, &acc);
    if (e == cudaSuccess) e = dmalloc(&h->n_active, 1, &acc);
    if (e == cudaSuccess) e = dmalloc(&h->max_count, 1, &acc);
    if (e == cudaSuccess) e = dmalloc(&h->act, P * h->I, &acc);
    if (e == cudaSuccess) e = dmalloc(&h->o, P * h->H, &acc);
    if (e == cudaSuccess) e = dmalloc(&h->x_stage, (size_t)max_T * h->H, &acc);
    if (e == cudaSuccess) e = dmalloc(&h->logits_stage, (size_t)max_T * h->E, &acc);
    if (e == cudaSuccess) e = dmalloc(&h->y_stage, (size_t)max_T * h->H, &acc);
    if (e == cudaSuccess) e = dmalloc(&h->dec_part, (size_t)h->sm_count * fe::kDecMaxT * h->H, &acc);
    if (e == cudaSuccess)
        e = cudaMemset(h->dec_part, 0, sizeof(unsigned long long) * (size_t)h->sm_count * fe::kDecMaxT * h->H);
    if (e == cudaSuccess) e = dmalloc(&h->dec_epoch, (size_t)h->sm_count + 1, &acc);
    if (e == cudaSuccess) e = dmalloc(&h->sg_table, 8 * (size_t)h->sm_count, &acc);
    if (e == cudaSuccess) e = cudaMemset(h->dec_epoch, 0, sizeof(unsigned long long) * ((size_t)h->sm_count + 1));
    if (e == cudaSuccess) e = dmalloc(&h->grp_bh, (P / fe::kGroupChunk + 1) * (size_t)h->E, &acc);
    {
        const size_t rt_floats = std::max((size_t)fe::kRtSplitFloats, (size_t)max_T * h->E);
        const size_t tiles = ((size_t)max_T + fe::kRtTok - 1) / fe::kRtTok;
        if (e == cudaSuccess) e = dmalloc(&h->rt_part, rt_floats, &acc);
        if (e == cudaSuccess) e = dmalloc(&h->rt_ticket, tiles, &acc);
        if (e == cudaSuccess) e = cudaMemset(h->rt_ticket, 0, sizeof(unsigned) * tiles);
    }
    // fp16 token and act rows (row-major for the tensor-core tiles, fragment
    // order for the streaming kernels: each forward writes before it reads)
    if (e == cudaSuccess) e = dmalloc(&h->tc_x, (size_t)max_T * h->H, &acc);
    if (e == cudaSuccess) e = dmalloc(&h->tc_xshift, (size_t)max_T, &acc);
    if (e == cudaSuccess) e = dmalloc(&h->tc_act, P * h->I, &acc);
    if (e == cudaSuccess) e = dmalloc(&h->tc_ashift, P, &acc);
    if (tc_shape_ok(h)) {
        if (e == cudaSuccess) e = dmalloc(&h->tc_tiles, 3 * tc_max_tiles(h, P), &acc);
        if (e == cudaSuccess) e = dmalloc(&h->tc_ntiles, 1, &acc);
    }
    if (h->nv_gu && e == cudaSuccess) e = nv_alloc_workspace(h, max_T, P, &acc);
    h->work_bytes = 0;
    for (auto& row : h->dec_planned)
        for (bool& b : row) b = false;
    if (e != cudaSuccess) {
        keep_status = h->status;
        h->status = nullptr;
        free_workspace(h);
        h->status = keep_status;
        return e == cudaErrorMemoryAllocation ? FE_ERR_OOM : FE_ERR_CUDA;
    }
    FE_CUDA_TRY(configure_kernels(h));
    h->max_T = max_T;
    h->max_k = max_top_k;
    h->work_bytes += acc;
    return FE_OK;
}

fe_status fe_moe_load_packed(fe_moe_t h, const uint8_t* gu_codes, const uint16_t* gu_scales, const uint8_t* dn_codes,
                             const uint16_t* dn_scales, int src_on_device, fe_stream_t stream)
{
    if (!h || !gu_codes || !gu_scales || !dn_codes || !dn_scales) return FE_ERR_INVALID_ARG;
    DeviceGuard g(h->device);
    if (!g.ok) return FE_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    const int64_t E = h->E, H = h->H, I = h->I;
    const size_t gu_c = (size_t)E * (H / 2) * (2 * I), gu_s = (size_t)E * (H / 32) * (2 * I);
    const size_t dn_c = (size_t)E * (I / 2) * H, dn_s = (size_t)E * (I / 32) * H;
    const uint8_t* sgc = gu_codes;
    const uint16_t* sgs = gu_scales;
    const uint8_t* sdc = dn_codes;
    const uint16_t* sds = dn_scales;
    void* staging = nullptr;
    if (!src_on_device) {
        const size_t bytes = gu_c + 2 * gu_s + dn_c + 2 * dn_s;
        FE_CUDA_TRY(cudaMallocAsync(&staging, bytes, s));
        uint8_t* b = static_cast<uint8_t*>(staging);
        FE_CUDA_TRY(cudaMemcpyAsync(b, gu_codes, gu_c, cudaMemcpyHostToDevice, s));
        FE_CUDA_TRY(cudaMemcpyAsync(b + gu_c, gu_scales, 2 * gu_s, cudaMemcpyHostToDevice, s));
        FE_CUDA_TRY(cudaMemcpyAsync(b + gu_c + 2 * gu_s, dn_codes, dn_c, cudaMemcpyHostToDevice, s));
        FE_CUDA_TRY(cudaMemcpyAsync(b + gu_c + 2 * gu_s + dn_c, dn_scales, 2 * dn_s, cudaMemcpyHostToDevice, s));
        sgc = b;
        sgs = reinterpret_cast<const uint16_t*>(b + gu_c);
        sdc = b + gu_c + 2 * gu_s;
        sds = reinterpret_cast<const uint16_t*>(b + gu_c + 2 * gu_s + dn_c);
    } else if (!aligned16(gu_codes) || !aligned16(gu_scales) || !aligned16(dn_codes) || !aligned16(dn_scales)) {
        return FE_ERR_INVALID_ARG;
    }
    fe::RelayoutParams rp{};
    rp.src_codes = sgc; rp.src_scales = sgs; rp.dst = h->gu_blocks;
    rp.E = E; rp.K = H; rp.N = 2 * I; rp.gate_up = 1;
    fe::relayout_kernel<<<1184, 256, 0, s>>>(rp);
    rp.src_codes = sdc; rp.src_scales = sds; rp.dst = h->dn_blocks;
    rp.K = I; rp.N = H; rp.gate_up = 0;
    fe::relayout_kernel<<<1184, 256, 0, s>>>(rp);
    fe::RowRelayoutParams rr{};
    rr.src_codes = sdc; rr.src_scales = sds; rr.dst = h->dn_rows;
    rr.E = E; rr.I = I; rr.H = H;
    fe::relayout_rows_kernel<<<1184, 256, 0, s>>>(rr);
    FE_CUDA_TRY(cudaGetLastError());
    // the tensor-core path needs every scale in the range where code x scale is an
    // exact f16; checked once here (this waits for the stream)
    h->tc_scales_ok = false;
    if (tc_shape_ok(h)) {
        uint32_t* bad = nullptr;
        FE_CUDA_TRY(cudaMallocAsync(reinterpret_cast<void**>(&bad), sizeof(uint32_t), s));
        FE_CUDA_TRY(cudaMemsetAsync(bad, 0, sizeof(uint32_t), s));
        fe::tc_scale_check_kernel<<<296, 256, 0, s>>>(sgs, gu_s, bad);
        fe::tc_scale_check_kernel<<<296, 256, 0, s>>>(sds, dn_s, bad);
        uint32_t hbad = 1;
        FE_CUDA_TRY(cudaMemcpyAsync(&hbad, bad, sizeof(uint32_t), cudaMemcpyDeviceToHost, s));
        FE_CUDA_TRY(cudaFreeAsync(bad, s));
        FE_CUDA_TRY(cudaStreamSynchronize(s));
        h->tc_scales_ok = hbad == 0;
    }
    if (staging) FE_CUDA_TRY(cudaFreeAsync(staging, s));
    h->loaded = true;
    return FE_OK;
}

fe_status fe_moe_load_nvfp4(fe_moe_t h, const uint8_t* gu_codes, const uint16_t* gu_scales, const uint8_t* dn_codes,
                            const uint16_t* dn_scales, int src_on_device, fe_stream_t stream)
{
    if (!h || !gu_codes || !gu_scales || !dn_codes || !dn_scales) return FE_ERR_INVALID_ARG;
    if (!nv_shape_ok(h)) return FE_ERR_UNSUPPORTED;
    DeviceGuard g(h->device);
    if (!g.ok) return FE_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    const int64_t E = h->E, H = h->H, I = h->I;
    const size_t gu_c = (size_t)E * (H / 2) * (2 * I), gu_s = (size_t)E * (H / 32) * (2 * I);
    const size_t dn_c = (size_t)E * (I / 2) * H, dn_s = (size_t)E * (I / 32) * H;
    const uint8_t* sgc = gu_codes;
    const uint16_t* sgs = gu_scales;
    const uint8_t* sdc = dn_codes;
    const uint16_t* sds = dn_scales;
    if (!h->nv_gu) {
        cudaError_t e = cudaSuccess;
        size_t acc = 0;
        if (e == cudaSuccess) e = dmalloc(&h->nv_gu, (size_t)E * (2 * I / fe::kNvM) * (H / fe::kNvKc) * fe::kNvAChunk, &acc);
        if (e == cudaSuccess) e = dmalloc(&h->nv_dn, (size_t)E * (H / fe::kNvM) * (I / fe::kNvKc) * fe::kNvAChunk, &acc);
        if (e == cudaSuccess) e = dmalloc(&h->nv_gug, (size_t)E * 2 * I, &acc);
        if (e == cudaSuccess) e = dmalloc(&h->nv_dng, (size_t)E * H, &acc);
        if (e == cudaSuccess && h->max_T > 0)
            e = nv_alloc_workspace(h, h->max_T, (size_t)h->max_T * h->max_k, &h->work_bytes);
        if (e != cudaSuccess) {
            void* ptrs[] = {h->nv_gu, h->nv_dn, h->nv_gug, h->nv_dng, h->nv_b, h->nv_bg, h->nv_xc, h->nv_xs, h->nv_xg};
            for (void* q : ptrs)
                if (q) cudaFree(q);
            h->nv_gu = h->nv_dn = h->nv_b = h->nv_xc = h->nv_xs = nullptr;
            h->nv_gug = h->nv_dng = h->nv_bg = h->nv_xg = nullptr;
            return record_cuda(e, "fe_moe_load_nvfp4 allocation");
        }
        h->weight_bytes += acc;
    }
    void* staging = nullptr;
    if (!src_on_device) {
        const size_t bytes = gu_c + 2 * gu_s + dn_c + 2 * dn_s;
        FE_CUDA_TRY(cudaMallocAsync(&staging, bytes, s));
        uint8_t* b = static_cast<uint8_t*>(staging);
        FE_CUDA_TRY(cudaMemcpyAsync(b, gu_codes, gu_c, cudaMemcpyHostToDevice, s));
        FE_CUDA_TRY(cudaMemcpyAsync(b + gu_c, gu_scales, 2 * gu_s, cudaMemcpyHostToDevice, s));
        FE_CUDA_TRY(cudaMemcpyAsync(b + gu_c + 2 * gu_s, dn_codes, dn_c, cudaMemcpyHostToDevice, s));
        FE_CUDA_TRY(cudaMemcpyAsync(b + gu_c + 2 * gu_s + dn_c, dn_scales, 2 * dn_s, cudaMemcpyHostToDevice, s));
        sgc = b;
        sgs = reinterpret_cast<const uint16_t*>(b + gu_c);
        sdc = b + gu_c + 2 * gu_s;
        sds = reinterpret_cast<const uint16_t*>(b + gu_c + 2 * gu_s + dn_c);
    }
    const long long n_gu = E * 2 * I, n_dn = E * H;
    fe::nvfp4_weights_kernel<<<(unsigned)((n_gu + 255) / 256), 256, 0, s>>>(sgc, sgs, (int)E, (int)H, (int)(2 * I), 1,
                                                                             (int)I, h->nv_gu, h->nv_gug);
    fe::nvfp4_weights_kernel<<<(unsigned)((n_dn + 255) / 256), 256, 0, s>>>(sdc, sds, (int)E, (int)I, (int)H, 0,
                                                                             (int)I, h->nv_dn, h->nv_dng);
    FE_CUDA_TRY(cudaGetLastError());
    if (staging) FE_CUDA_TRY(cudaFreeAsync(staging, s));
    return FE_OK;
}

fe_status fe_moe_nvfp4_quantize_device(const float* src, int64_t rows, int64_t K, uint8_t* codes, uint8_t* sf,
                                       float* row_scale, fe_stream_t stream)
{
    if (!src || !codes || !sf || !row_scale || rows < 0 || K < 16 || K % 16 || rows > (int64_t)1 << 26 ||
        K > (int64_t)1 << 20 || !aligned16(src) || (reinterpret_cast<uintptr_t>(codes) & 7u) ||
        (reinterpret_cast<uintptr_t>(row_scale) & 3u))
        return FE_ERR_INVALID_ARG;
    if (rows == 0) return FE_OK;
    fe::nvfp4_rows_kernel<false><<<(unsigned)((rows * 32 + 255) / 256), 256, 0, (cudaStream_t)stream>>>(
        src, (int)rows, (int)K, codes, sf, row_scale);
    return cudaGetLastError() == cudaSuccess ? FE_OK : FE_ERR_CUDA;
}

fe_status fe_moe_load_int2(fe_moe_t h, const uint8_t* formats, const uint8_t* gu_codes, const uint16_t* gu_scales,
                           const uint8_t* dn_codes, const uint16_t* dn_scales, int src_on_device, fe_stream_t stream)
{
    if (!h || !formats || !gu_codes || !gu_scales || !dn_codes || !dn_scales) return FE_ERR_INVALID_ARG;
    if (h->H % 64 != 0 || h->I % 64 != 0) return FE_ERR_UNSUPPORTED;
    DeviceGuard g(h->device);
    if (!g.ok) return FE_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    const int64_t E = h->E, H = h->H, I = h->I;
    const size_t gu_c = (size_t)E * (H / 4) * (2 * I), gu_s = (size_t)E * (H / 32) * (2 * I);
    const size_t dn_c = (size_t)E * (I / 4) * H, dn_s = (size_t)E * (I / 32) * H;
    if (!h->gu2_blocks) {
        cudaError_t e = cudaSuccess;
        size_t acc = 0;
        if (e == cudaSuccess) e = dmalloc(&h->fmt, (size_t)E, &acc);
        if (e == cudaSuccess) e = dmalloc(&h->gu2_blocks, (size_t)E * (I / 16) * 2 * fe::int2_block_bytes((int)H), &acc);
        if (e == cudaSuccess) e = dmalloc(&h->dn2_rows, (size_t)E * (I / 32) * 10 * (size_t)H, &acc);
        if (e != cudaSuccess) return e == cudaErrorMemoryAllocation ? FE_ERR_OOM : FE_ERR_CUDA;
        h->weight_bytes += acc;
    }
    const uint8_t* sgc = gu_codes;
    const uint16_t* sgs = gu_scales;
    const uint8_t* sdc = dn_codes;
    const uint16_t* sds = dn_scales;
    void* staging = nullptr;
    if (!src_on_device) {
        const size_t bytes = gu_c + 2 * gu_s + dn_c + 2 * dn_s;
        FE_CUDA_TRY(cudaMallocAsync(&staging, bytes, s));
        uint8_t* b = static_cast<uint8_t*>(staging);
        FE_CUDA_TRY(cudaMemcpyAsync(b, gu_codes, gu_c, cudaMemcpyHostToDevice, s));
        FE_CUDA_TRY(cudaMemcpyAsync(b + gu_c, gu_scales, 2 * gu_s, cudaMemcpyHostToDevice, s));
        FE_CUDA_TRY(cudaMemcpyAsync(b + gu_c + 2 * gu_s, dn_codes, dn_c, cudaMemcpyHostToDevice, s));
        FE_CUDA_TRY(cudaMemcpyAsync(b + gu_c + 2 * gu_s + dn_c, dn_scales, 2 * dn_s, cudaMemcpyHostToDevice, s));
        sgc = b;
        sgs = reinterpret_cast<const uint16_t*>(b + gu_c);
        sdc = b + gu_c + 2 * gu_s;
        sds = reinterpret_cast<const uint16_t*>(b + gu_c + 2 * gu_s + dn_c);
    }
    bool any = false;
    for (int64_t e = 0; e < E; ++e) any |= formats[e] != 0;
    FE_CUDA_TRY(cudaMemcpyAsync(h->fmt, formats, (size_t)E, cudaMemcpyHostToDevice, s));
    fe::RelayoutParams rp{};
    rp.src_codes = sgc; rp.src_scales = sgs; rp.dst = h->gu2_blocks;
    rp.E = E; rp.K = H; rp.N = 2 * I; rp.gate_up = 1;
    fe::relayout_int2_kernel<<<1184, 256, 0, s>>>(rp);
    fe::RowRelayoutParams rr{};
    rr.src_codes = sdc; rr.src_scales = sds; rr.dst = h->dn2_rows;
    rr.E = E; rr.I = I; rr.H = H;
    fe::relayout_int2_rows_kernel<<<1184, 256, 0, s>>>(rr);
    FE_CUDA_TRY(cudaGetLastError());
    if (staging) FE_CUDA_TRY(cudaFreeAsync(staging, s));
    // the host's format table and buffers are read by the copies: wait before returning
    FE_CUDA_TRY(cudaStreamSynchronize(s));
    h->has_int2 = any;
    return FE_OK;
}

}  // extern "C"

namespace {

// The body of fe_moe_forward (also run by the stack for each of its layers).
fe_status forward_impl(fe_moe_t h, const void* x_bf16, const float* router_logits, int T, int top_k, void* y_bf16,
                       fe_stream_t stream)
{
    if (!h || T < 0 || top_k < 1 || top_k > h->E) return FE_ERR_INVALID_ARG;
    if (T == 0) return FE_OK;
    if (!x_bf16 || !router_logits || !y_bf16 || x_bf16 == y_bf16) return FE_ERR_INVALID_ARG;
    if (!h->loaded) return FE_ERR_NOT_LOADED;
    if (T > h->max_T || top_k > h->max_k) return FE_ERR_CAPACITY;
    if ((reinterpret_cast<uintptr_t>(x_bf16) & 3u) || (reinterpret_cast<uintptr_t>(y_bf16) & 3u) ||
        (reinterpret_cast<uintptr_t>(router_logits) & 3u))
        return FE_ERR_INVALID_ARG;
    const bool tc_ok = tc_shape_ok(h) && h->tc_scales_ok && h->tc_x != nullptr;
    if (h->path == FE_PATH_TCGEN05 && !tc_ok) return FE_ERR_UNSUPPORTED;
    DeviceGuard g(h->device);
    if (!g.ok) return FE_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    const int P = T * top_k;

    if (h->path == FE_PATH_AUTO || h->path == FE_PATH_FUSED_DECODE) {
        const uint32_t wbytes = decode_weight_bytes(h, T, top_k);
        if (wbytes > 0) {
            fe_status st = decode_path(h, x_bf16, router_logits, T, top_k, y_bf16, wbytes, s);
            if (st == FE_OK) {
                h->last_T = T;
                h->last_k = top_k;
                h->last_path = FE_PATH_FUSED_DECODE;
                h->last_kernels = 1;
            }
            return st;
        }
        if (h->path == FE_PATH_FUSED_DECODE) return FE_ERR_UNSUPPORTED;
    }
    // INT2 experts are read by the single-launch decode kernel only
    if (h->has_int2) return FE_ERR_UNSUPPORTED;
    if (h->path == FE_PATH_NVFP4) {
        if (!h->nv_gu || !h->nv_b || !h->tc_tiles) return FE_ERR_UNSUPPORTED;
        if (!aligned16(x_bf16)) return FE_ERR_INVALID_ARG;   // the x rows are read in 16-byte pieces
        const fe_status rs = route_and_group(h, router_logits, T, top_k, nullptr, s);
        if (rs != FE_OK) return rs;
        const fe_status st = nvfp4_path(h, static_cast<const uint16_t*>(x_bf16), T, top_k, s);
        if (st != FE_OK) return st;
        dim3 cgrid((h->H / 8 + 255) / 256, T);
        fe::combine_kernel<true><<<cgrid, 256, 0, s>>>(h->o, h->w, h->pair_row, h->H, top_k,
                                                        static_cast<__nv_bfloat16*>(y_bf16));
        FE_CUDA_TRY(cudaGetLastError());
        h->last_T = T;
        h->last_k = top_k;
        h->last_path = FE_PATH_NVFP4;
        const bool large_route = T >= kRouteLargeTokens && fe::route_large_ok(h->E, top_k);
        h->last_kernels = (large_route ? 4 : 1) + 6 + 1;   // routing, tile list, x rows, 2 x (images, tiles), combine
        return FE_OK;
    }

    const bool use_tc = tc_ok && (h->path == FE_PATH_TCGEN05 || (h->path == FE_PATH_AUTO && P >= kTcAutoPairs));
    SgSetup sg;
    const bool use_stream = !use_tc && stream_setup(h, T, sg);
    {
        const fe_status rs = route_and_group(h, router_logits, T, top_k, use_stream ? &sg.split : nullptr, s);
        if (rs != FE_OK) return rs;
    }
    fe_status st = FE_OK;
    if (use_tc)
        st = tcgen05_path(h, static_cast<const uint16_t*>(x_bf16), T, top_k, s);
    else if (use_stream)
        st = stream_path(h, static_cast<const uint16_t*>(x_bf16), top_k, sg, s);
    else
        st = gemv_path(h, static_cast<const uint16_t*>(x_bf16), T, top_k, s);
    if (st != FE_OK) return st;

    dim3 cgrid((h->H / 8 + 255) / 256, T);
    if (use_tc)   // the tensor-core down tiles leave o as bf16
        fe::combine_kernel<true><<<cgrid, 256, 0, s>>>(h->o, h->w, h->pair_row, h->H, top_k,
                                                        static_cast<__nv_bfloat16*>(y_bf16));
    else
        fe::combine_kernel<false><<<cgrid, 256, 0, s>>>(h->o, h->w, h->pair_row, h->H, top_k,
                                              static_cast<__nv_bfloat16*>(y_bf16));
    FE_CUDA_TRY(cudaGetLastError());
    h->last_T = T;
    h->last_k = top_k;
    h->last_path = use_tc ? FE_PATH_TCGEN05 : FE_PATH_GEMV;
    const bool large_route = T >= kRouteLargeTokens && fe::route_large_ok(h->E, top_k);
    h->last_kernels = (large_route ? 4 : 1) + (use_tc ? 6 : 2) + 1;   // routing, projections, combine
    return FE_OK;
}

// The router GEMM fused with the top-k (router.cuh).
fe_status router_impl(fe_moe_s* h, const void* x_bf16, const void* w_router_bf16, int T, int top_k, float* logits,
                      int32_t* idx, float* w, cudaStream_t s)
{
    if (!h || T < 0 || top_k < 1 || top_k > h->E) return FE_ERR_INVALID_ARG;
    if (T == 0) return FE_OK;
    if (!x_bf16 || !w_router_bf16 || !logits) return FE_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(x_bf16) | reinterpret_cast<uintptr_t>(w_router_bf16)) & 15u) return FE_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(logits) & 3u) return FE_ERR_INVALID_ARG;
    const int J = h->E <= 32 ? 1 : h->E <= 64 ? 2 : h->E <= 128 ? 4 : h->E <= 256 ? 8 : 16;
    if (h->H % 64 != 0 || h->E > 512 || top_k > fe::kRtMaxK || top_k * J > fe::kRtCand) return FE_ERR_UNSUPPORTED;
    if (!h->rt_part || T > h->max_T) return FE_ERR_CAPACITY;
    fe::RouterParams rp;
    rp.x = static_cast<const uint16_t*>(x_bf16);
    rp.wr = static_cast<const uint16_t*>(w_router_bf16);
    rp.T = T;
    rp.H = h->H;
    rp.E = h->E;
    rp.k = top_k;
    rp.ks = fe::router_splits(T, h->H, h->E);
    rp.part = h->rt_part;
    rp.ticket = h->rt_ticket;
    rp.logits = logits;
    rp.idx = idx;
    rp.w = w;
    rp.status = h->status;
    const dim3 grid((T + fe::kRtTok - 1) / fe::kRtTok, (h->E + fe::kRtExp - 1) / fe::kRtExp, rp.ks);
    fe::router_kernel<<<grid, fe::kRtThreads, 0, s>>>(rp);
    FE_CUDA_TRY(cudaGetLastError());
    return FE_OK;
}

}  // namespace

extern "C" {

fe_status fe_moe_router(fe_moe_t h, const void* x_bf16, const void* w_router_bf16, int T, int top_k, float* logits,
                        int32_t* idx, float* w, fe_stream_t stream)
{
    if (!h) return FE_ERR_INVALID_ARG;
    DeviceGuard g(h->device);
    if (!g.ok) return FE_ERR_CUDA;
    return router_impl(h, x_bf16, w_router_bf16, T, top_k, logits, idx, w, (cudaStream_t)stream);
}

fe_status fe_moe_forward_router(fe_moe_t h, const void* x_bf16, const void* w_router_bf16, int T, int top_k,
                                void* y_bf16, float* logits, fe_stream_t stream)
{
    if (!h) return FE_ERR_INVALID_ARG;
    if (T > 0 && !h->loaded) return FE_ERR_NOT_LOADED;
    DeviceGuard g(h->device);
    if (!g.ok) return FE_ERR_CUDA;
    const fe_status st = router_impl(h, x_bf16, w_router_bf16, T, top_k, logits, nullptr, nullptr,
                                     (cudaStream_t)stream);
    if (st != FE_OK) return st;
    return forward_impl(h, x_bf16, logits, T, top_k, y_bf16, stream);
}

fe_status fe_moe_forward(fe_moe_t h, const void* x_bf16, const float* router_logits, int T, int top_k, void* y_bf16,
                         fe_stream_t stream)
{
    return forward_impl(h, x_bf16, router_logits, T, top_k, y_bf16, stream);
}

fe_status fe_moe_forward_host(fe_moe_t h, const uint16_t* x_host, const float* logits_host, int T, int top_k,
                              uint16_t* y_host, fe_stream_t stream)
{
    if (!h || T < 0 || top_k < 1 || top_k > h->E) return FE_ERR_INVALID_ARG;
    if (T == 0) return FE_OK;
    if (!x_host || !logits_host || !y_host) return FE_ERR_INVALID_ARG;
    if (!h->loaded) return FE_ERR_NOT_LOADED;
    if (T > h->max_T || top_k > h->max_k) return FE_ERR_CAPACITY;
    DeviceGuard g(h->device);
    if (!g.ok) return FE_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    FE_CUDA_TRY(cudaMemcpyAsync(h->x_stage, x_host, sizeof(uint16_t) * (size_t)T * h->H, cudaMemcpyHostToDevice, s));
    FE_CUDA_TRY(cudaMemcpyAsync(h->logits_stage, logits_host, sizeof(float) * (size_t)T * h->E,
                                cudaMemcpyHostToDevice, s));
    fe_status st = fe_moe_forward(h, h->x_stage, h->logits_stage, T, top_k, h->y_stage, stream);
    if (st != FE_OK) return st;
    FE_CUDA_TRY(cudaMemcpyAsync(y_host, h->y_stage, sizeof(uint16_t) * (size_t)T * h->H, cudaMemcpyDeviceToHost, s));
    FE_CUDA_TRY(cudaStreamSynchronize(s));
    return FE_OK;
}

fe_status fe_moe_stack_create(const fe_moe_t* layers, int n_layers, fe_moe_stack_t* out)
{
    if (!out) return FE_ERR_INVALID_ARG;
    *out = nullptr;
    if (!layers || n_layers < 1) return FE_ERR_INVALID_ARG;
    for (int l = 0; l < n_layers; ++l) {
        const fe_moe_s* h = layers[l];
        if (!h || h->E != layers[0]->E || h->H != layers[0]->H || h->device != layers[0]->device)
            return FE_ERR_INVALID_ARG;
        if (!h->loaded) return FE_ERR_NOT_LOADED;
        if (h->max_T < 1) return FE_ERR_CAPACITY;
    }
    fe_moe_stack_s* st = new (std::nothrow) fe_moe_stack_s();
    if (!st) return FE_ERR_OOM;
    st->layers.assign(layers, layers + n_layers);
    st->device = layers[0]->device;
    st->E = layers[0]->E;
    st->H = layers[0]->H;
    st->max_T = layers[0]->max_T;
    for (int l = 1; l < n_layers; ++l) st->max_T = std::min(st->max_T, layers[l]->max_T);
    DeviceGuard g(st->device);
    cudaError_t e = g.ok ? cudaSuccess : cudaErrorInvalidDevice;
    const size_t row = (size_t)st->max_T * st->H;
    if (e == cudaSuccess) e = dmalloc(&st->a_stage, ((size_t)n_layers + 1) * row, nullptr);
    if (e == cudaSuccess) e = dmalloc(&st->b_stage, (size_t)n_layers * row, nullptr);
    if (e == cudaSuccess) e = dmalloc(&st->logits_stage, (size_t)n_layers * st->max_T * st->E, nullptr);
    // the persistent launches (one token each): every layer of one shape, small enough, the
    // kernel resident on every SM
    st->sm_count = layers[0]->sm_count;
    bool same = true;
    for (int l = 1; l < n_layers; ++l) same &= layers[l]->I == layers[0]->I;
    const int H = st->H, I = layers[0]->I;
    if (e == cudaSuccess && same && n_layers <= fe::kStkMaxLayers && st->E <= fe::kDecMaxE && H <= fe::kDecMaxH &&
        I <= 1024 && st->sm_count <= fe::kDecMaxCtas) {
        const uint32_t smem = fe::stack_smem_layout(H).total;
        int per_sm = 0;
        if (smem <= (uint32_t)layers[0]->smem_optin &&
            cudaFuncSetAttribute(fe::stack_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) ==
                cudaSuccess &&
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fe::stack_decode_kernel, fe::kStkThreads, smem) ==
                cudaSuccess &&
            per_sm >= 1) {
            st->stk_smem = smem;
            st->h_layers.resize(n_layers);
            for (int l = 0; l < n_layers; ++l) {
                fe_moe_s* h = layers[l];
                st->h_layers[l] = fe::StackLayer{h->gu_blocks, h->dn_rows, h->idx, h->w, h->counts, h->offsets,
                                                 h->sorted_pair, h->pair_row};
            }
            const size_t pbytes = sizeof(unsigned long long) * fe::kStkBufs * (size_t)st->sm_count * H;
            e = cudaMalloc(reinterpret_cast<void**>(&st->part), pbytes);
            if (e == cudaSuccess) e = cudaMemset(st->part, 0, pbytes);
            if (e == cudaSuccess) e = dmalloc(&st->ctr, (size_t)st->sm_count + 2 * fe::kStkBufs, nullptr);
            if (e == cudaSuccess) e = cudaMemset(st->ctr, 0, sizeof(unsigned long long) * ((size_t)st->sm_count + 2 * fe::kStkBufs));
            if (e == cudaSuccess) e = dmalloc(&st->d_layers, (size_t)n_layers, nullptr);
            if (e == cudaSuccess)
                e = cudaMemcpy(st->d_layers, st->h_layers.data(), sizeof(fe::StackLayer) * n_layers,
                               cudaMemcpyHostToDevice);
            st->persistent_ok = e == cudaSuccess;
        } else {
            cudaGetLastError();   // a refused attribute leaves no error behind
        }
    }
    if (e != cudaSuccess) {
        fe_moe_stack_destroy(st);
        return record_cuda(e, "fe_moe_stack_create");
    }
    *out = st;
    return FE_OK;
}

}  // extern "C"

namespace {

// Whether fe_moe_stack_forward can run the stack on the persistent kernel, which
// computes one token per launch: a call at T = 1, or at a few tokens whose routing
// is sparse (T * top_k at most a quarter of E, so the tokens rarely share an expert
// and a launch per token reads about the bytes one launch for all would), runs as T
// launches.  Also needed: every layer on the single-launch decode kernel's shapes
// at one token, E2M1 experts only, the layers' buffers unchanged since the stack
// was made, and x / y either chained (y = x + T*H) or disjoint.  Returns 1
// (independent), 2 (chained) or 0.
int stack_persistent_mode(fe_moe_stack_s* st, const void* x, void* y, int T, int top_k)
{
    if (!st->persistent_ok || !st->prefetch || top_k > fe::kStkMaxK) return 0;
    if (T != 1 && (T > fe::kStkMaxTokens || 4 * T * top_k > st->E)) return 0;
    const int n = (int)st->layers.size();
    for (int l = 0; l < n; ++l) {
        fe_moe_s* h = st->layers[l];
        if (h->path != FE_PATH_AUTO && h->path != FE_PATH_FUSED_DECODE) return 0;
        if (h->has_int2) return 0;   // the persistent kernel reads E2M1 experts only
        if (decode_weight_bytes(h, 1, top_k) == 0) return 0;
        const fe::StackLayer& s = st->h_layers[l];
        if (s.gu_blocks != h->gu_blocks || s.dn_rows != h->dn_rows || s.idx != h->idx || s.w != h->w ||
            s.counts != h->counts || s.offsets != h->offsets || s.sorted_pair != h->sorted_pair ||
            s.pair_row != h->pair_row)
            return 0;
    }
    const size_t bytes = sizeof(uint16_t) * (size_t)n * T * st->H;
    const char* xb = static_cast<const char*>(x);
    const char* yb = static_cast<const char*>(y);
    if (yb == xb + sizeof(uint16_t) * (size_t)T * st->H) return 2;
    if (yb + bytes <= xb || xb + bytes <= yb) return 1;
    return 0;
}

fe_status stack_persistent_launch(fe_moe_stack_s* st, const void* x, const float* logits, int T, int top_k,
                                  void* y, int mode, cudaStream_t s)
{
    fe_moe_s* h0 = st->layers[0];
    fe::StackParams sp{};
    sp.layers = st->d_layers;
    sp.L = (int)st->layers.size();
    sp.E = st->E; sp.H = st->H; sp.I = h0->I; sp.k = top_k;
    sp.T = T;
    sp.ldx = (size_t)T * st->H;
    sp.ldl = (size_t)T * st->E;
    sp.ldy = (size_t)T * st->H;
    sp.chained = mode == 2;
    sp.part = st->part;
    sp.ctr = st->ctr;
    sp.status = h0->status;
    sp.timeout_ns = 200ull * 1000 * 1000;
    sp.trace = h0->trace;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(st->sm_count);
    cfg.blockDim = dim3(fe::kStkThreads);
    cfg.dynamicSmemBytes = st->stk_smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    for (int t = 0; t < T; ++t) {   // one launch per token: rows t of every layer
        sp.t = t;
        sp.x = static_cast<const uint16_t*>(x) + (size_t)t * st->H;
        sp.logits = logits + (size_t)t * st->E;
        sp.y = static_cast<uint16_t*>(y) + (size_t)t * st->H;
        FE_CUDA_TRY(cudaLaunchKernelEx(&cfg, fe::stack_decode_kernel, sp));
    }
    for (fe_moe_s* h : st->layers) {
        h->last_T = T;
        h->last_k = top_k;
        h->last_path = FE_PATH_FUSED_DECODE;
        h->last_kernels = 0;
    }
    st->last_launches = T;
    return FE_OK;
}

}  // namespace

extern "C" {

fe_status fe_moe_stack_forward(fe_moe_stack_t st, const void* x_bf16, const float* logits, int T, int top_k,
                               void* y_bf16, fe_stream_t stream)
{
    if (!st || T < 0 || top_k < 1) return FE_ERR_INVALID_ARG;
    if (T == 0) return FE_OK;
    if (!x_bf16 || !logits || !y_bf16) return FE_ERR_INVALID_ARG;
    const size_t row_bytes = sizeof(uint16_t) * (size_t)T * st->H;
    const uintptr_t xa = reinterpret_cast<uintptr_t>(x_bf16), ya = reinterpret_cast<uintptr_t>(y_bf16);
    if ((xa > ya ? xa - ya : ya - xa) < row_bytes) return FE_ERR_INVALID_ARG;   // y_l would overlap x_l
    if ((xa & 3u) || (ya & 3u) || (reinterpret_cast<uintptr_t>(logits) & 3u)) return FE_ERR_INVALID_ARG;
    // every layer's arguments are checked before the first launch
    for (fe_moe_s* h : st->layers) {
        if (top_k > h->E) return FE_ERR_INVALID_ARG;
        if (!h->loaded) return FE_ERR_NOT_LOADED;
        if (T > h->max_T || top_k > h->max_k) return FE_ERR_CAPACITY;
        if (h->path == FE_PATH_TCGEN05 && !(tc_shape_ok(h) && h->tc_scales_ok && h->tc_x)) return FE_ERR_UNSUPPORTED;
    }
    const int n = (int)st->layers.size();
    const size_t xe = (size_t)T * st->H;
    const int mode = stack_persistent_mode(st, x_bf16, y_bf16, T, top_k);
    if (mode > 0) {
        DeviceGuard g(st->device);
        if (!g.ok) return FE_ERR_CUDA;
        return stack_persistent_launch(st, x_bf16, logits, T, top_k, y_bf16, mode, (cudaStream_t)stream);
    }
    int launches = 0;
    for (int l = 0; l < n; ++l) {
        const fe_status r = forward_impl(st->layers[l], static_cast<const uint16_t*>(x_bf16) + l * xe,
                                         logits + (size_t)l * T * st->E, T, top_k,
                                         static_cast<uint16_t*>(y_bf16) + l * xe, stream);
        if (r != FE_OK) return r;
        launches += st->layers[l]->last_kernels;
    }
    st->last_launches = launches;
    return FE_OK;
}

fe_status fe_moe_stack_forward_host(fe_moe_stack_t st, const uint16_t* x_host, const float* logits_host, int T,
                                    int top_k, uint16_t* y_host, int chained, fe_stream_t stream)
{
    if (!st || T < 0 || top_k < 1) return FE_ERR_INVALID_ARG;
    if (T == 0) return FE_OK;
    if (!x_host || !logits_host || !y_host) return FE_ERR_INVALID_ARG;
    if (T > st->max_T) return FE_ERR_CAPACITY;
    DeviceGuard g(st->device);
    if (!g.ok) return FE_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    const size_t n = st->layers.size();
    const size_t row = sizeof(uint16_t) * (size_t)T * st->H;
    const size_t xs = chained ? row : n * row;
    FE_CUDA_TRY(cudaMemcpyAsync(st->a_stage, x_host, xs, cudaMemcpyHostToDevice, s));
    FE_CUDA_TRY(cudaMemcpyAsync(st->logits_stage, logits_host, sizeof(float) * n * T * st->E, cudaMemcpyHostToDevice, s));
    uint16_t* y_dev = chained ? st->a_stage + (size_t)T * st->H : st->b_stage;
    const fe_status r = fe_moe_stack_forward(st, st->a_stage, st->logits_stage, T, top_k, y_dev, stream);
    if (r != FE_OK) return r;
    const uint16_t* y_src = chained ? st->a_stage + n * (size_t)T * st->H : st->b_stage;
    FE_CUDA_TRY(cudaMemcpyAsync(y_host, y_src, xs, cudaMemcpyDeviceToHost, s));
    FE_CUDA_TRY(cudaStreamSynchronize(s));
    return FE_OK;
}

fe_status fe_moe_stack_set_prefetch(fe_moe_stack_t st, int on)
{
    if (!st) return FE_ERR_INVALID_ARG;
    st->prefetch = on != 0;
    return FE_OK;
}

int fe_moe_stack_last_launches(fe_moe_stack_t st) { return st ? st->last_launches : -1; }

void fe_moe_stack_destroy(fe_moe_stack_t st)
{
    if (!st) return;
    {
        DeviceGuard g(st->device);
        cudaDeviceSynchronize();
        if (st->part) cudaFree(st->part);
        if (st->ctr) cudaFree(st->ctr);
        if (st->d_layers) cudaFree(st->d_layers);
        if (st->a_stage) cudaFree(st->a_stage);
        if (st->b_stage) cudaFree(st->b_stage);
        if (st->logits_stage) cudaFree(st->logits_stage);
    }
    delete st;
}

fe_status fe_moe_get_routing(fe_moe_t h, int32_t* idx, float* w, int32_t* offsets, int32_t* sorted_pair,
                             fe_stream_t stream)
{
    if (!h) return FE_ERR_INVALID_ARG;
    if (!h->idx) return FE_ERR_CAPACITY;
    DeviceGuard g(h->device);
    if (!g.ok) return FE_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    const size_t P = (size_t)h->last_T * h->last_k;
    if (idx && P) FE_CUDA_TRY(cudaMemcpyAsync(idx, h->idx, sizeof(int32_t) * P, cudaMemcpyDeviceToDevice, s));
    if (w && P) FE_CUDA_TRY(cudaMemcpyAsync(w, h->w, sizeof(float) * P, cudaMemcpyDeviceToDevice, s));
    if (offsets)
        FE_CUDA_TRY(cudaMemcpyAsync(offsets, h->offsets, sizeof(int32_t) * (h->E + 1), cudaMemcpyDeviceToDevice, s));
    if (sorted_pair && P)
        FE_CUDA_TRY(cudaMemcpyAsync(sorted_pair, h->sorted_pair, sizeof(int32_t) * P, cudaMemcpyDeviceToDevice, s));
    return FE_OK;
}

fe_status fe_moe_get_grouping(fe_moe_t h, int32_t* counts, int32_t* pair_row, fe_stream_t stream)
{
    if (!h) return FE_ERR_INVALID_ARG;
    if (!h->idx) return FE_ERR_CAPACITY;
    DeviceGuard g(h->device);
    if (!g.ok) return FE_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    const size_t P = (size_t)h->last_T * h->last_k;
    if (counts) FE_CUDA_TRY(cudaMemcpyAsync(counts, h->counts, sizeof(int32_t) * h->E, cudaMemcpyDeviceToDevice, s));
    if (pair_row && P)
        FE_CUDA_TRY(cudaMemcpyAsync(pair_row, h->pair_row, sizeof(int32_t) * P, cudaMemcpyDeviceToDevice, s));
    return FE_OK;
}

fe_status fe_moe_get_status(fe_moe_t h, uint32_t* bits)
{
    if (!h) return FE_ERR_INVALID_ARG;
    DeviceGuard g(h->device);
    if (!g.ok) return FE_ERR_CUDA;
    uint32_t v = 0;
    FE_CUDA_TRY(cudaDeviceSynchronize());
    FE_CUDA_TRY(cudaMemcpy(&v, h->status, sizeof(v), cudaMemcpyDeviceToHost));
    FE_CUDA_TRY(cudaMemset(h->status, 0, sizeof(v)));
    if (bits) *bits = v;
    return v ? FE_ERR_DEVICE_STATUS : FE_OK;
}

fe_status fe_moe_set_path(fe_moe_t h, int path)
{
    if (!h || path < FE_PATH_AUTO || path > FE_PATH_NVFP4) return FE_ERR_INVALID_ARG;
    h->path = path;
    return FE_OK;
}

fe_status fe_moe_set_exchange_test(fe_moe_t h, int unreachable, unsigned long long wait_ns)
{
    if (!h || wait_ns == 0) return FE_ERR_INVALID_ARG;
    h->test_extra_arrivals = unreachable ? 1 : 0;
    h->exchange_timeout_ns = unreachable ? wait_ns : 200ull * 1000 * 1000;
    return FE_OK;
}

fe_status fe_moe_set_trace(fe_moe_t h, unsigned long long* device_buf)
{
    if (!h) return FE_ERR_INVALID_ARG;
    h->trace = device_buf;
    return FE_OK;
}

fe_status fe_moe_last_forward_info(fe_moe_t h, int* path, int* kernels)
{
    if (!h) return FE_ERR_INVALID_ARG;
    if (path) *path = h->last_path;
    if (kernels) *kernels = h->last_kernels;
    return FE_OK;
}

void fe_moe_destroy(fe_moe_t h)
{
    if (!h) return;
    {
        DeviceGuard g(h->device);
        cudaDeviceSynchronize();
        free_workspace(h);
        void* ptrs[] = {h->gu_blocks, h->dn_blocks, h->dn_rows, h->fmt, h->gu2_blocks, h->dn2_rows,
                        h->nv_gu, h->nv_dn, h->nv_gug, h->nv_dng};
        for (void* p : ptrs)
            if (p) cudaFree(p);
    }
    delete h;
}

size_t fe_moe_device_bytes(fe_moe_t h) { return h ? h->weight_bytes + h->work_bytes : 0; }

const char* fe_moe_last_error(void) { return g_last_error; }

fe_status fe_moe_pack_host(const float* W, int64_t E, int64_t K, int64_t N, uint8_t* codes, uint16_t* scales)
{
    if (!W || !codes || !scales || E < 1 || K < 32 || N < 1 || K % 32) return FE_ERR_INVALID_ARG;
    fe_host::pack(W, E, K, N, codes, scales);
    return FE_OK;
}

fe_status fe_moe_pack_int2_host(const float* W, int64_t E, int64_t K, int64_t N, uint8_t* codes,
                                uint16_t* scales)
{
    if (!W || !codes || !scales || E < 1 || K < 32 || N < 1 || K % 32) return FE_ERR_INVALID_ARG;
    fe_host::pack_int2(W, E, K, N, codes, scales);
    return FE_OK;
}

fe_status fe_moe_pack_int2_device(const float* W, int64_t E, int64_t K, int64_t N, uint8_t* codes, uint16_t* scales,
                                  fe_stream_t stream)
{
    if (!W || !codes || !scales || E < 1 || K < 32 || N < 1 || K % 32) return FE_ERR_INVALID_ARG;
    const int64_t total = E * (K / 32) * N;
    const int64_t blocks = std::min<int64_t>((total + 255) / 256, 148 * 32);
    fe::pack_int2_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(W, E, K, N, codes, scales);
    return cudaGetLastError() == cudaSuccess ? FE_OK : FE_ERR_CUDA;
}

fe_status fe_moe_pack_device(const float* W, int64_t E, int64_t K, int64_t N, uint8_t* codes, uint16_t* scales,
                             fe_stream_t stream)
{
    if (!W || !codes || !scales || E < 1 || K < 32 || N < 1 || K % 32) return FE_ERR_INVALID_ARG;
    const int64_t total = E * (K / 32) * N;
    const int64_t blocks = std::min<int64_t>((total + 255) / 256, 148 * 32);
    fe::pack_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(W, E, K, N, codes, scales);
    return cudaGetLastError() == cudaSuccess ? FE_OK : FE_ERR_CUDA;
}


// ---------------------------------------------------------------------------
// Allocation-free forward (fe_moe_forward_noalloc).
//
// For callers that may not allocate device memory at all -- no cudaMalloc,
// no stream-ordered pool, no library that allocates on their behalf -- for
// instance code that runs under an external memory manager that owns every
// device byte, or inside a region where an allocation could stall or fail.
// Such a caller passes the packed weights, x, the logits and y in its own
// buffers; the routing lists, act and the per-pair down outputs live in one
// file-scope device array instead of a reserved workspace.
// ---------------------------------------------------------------------------
}  // extern "C"

namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)4 << 20;   // 4 MiB, held by every GPU that loads the library
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

struct NoAllocDevice {
    bool ready = false;
    unsigned char* scratch = nullptr;   // device address of g_noalloc_scratch on this device
};
std::mutex g_noalloc_mu;
NoAllocDevice g_noalloc_dev[64];

// Once per device, with that device current: the device address of the
// scratch array (its name in host code is only a stand-in) and the kernels'
// shared-memory opt-in.  Neither allocates.
fe_status noalloc_setup(int dev, unsigned char** scratch)
{
    if (dev < 0 || dev >= 64) return FE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    NoAllocDevice& d = g_noalloc_dev[dev];
    if (!d.ready) {
        void* ptr = nullptr;
        FE_CUDA_TRY(cudaGetSymbolAddress(&ptr, g_noalloc_scratch));
        int optin = 0;
        FE_CUDA_TRY(cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev));
        FE_CUDA_TRY(cudaFuncSetAttribute(fe::route_group_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, optin));
        FE_CUDA_TRY(cudaFuncSetAttribute(fe::gemv_canonical_kernel<1, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin));
        FE_CUDA_TRY(cudaFuncSetAttribute(fe::gemv_canonical_kernel<4, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin));
        FE_CUDA_TRY(cudaFuncSetAttribute(fe::gemv_canonical_kernel<1, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin));
        FE_CUDA_TRY(cudaFuncSetAttribute(fe::gemv_canonical_kernel<4, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin));
        d.scratch = static_cast<unsigned char*>(ptr);
        d.ready = true;
    }
    *scratch = d.scratch;
    return FE_OK;
}

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

// Carve the scratch array; returns the bytes needed (0 = does not fit).
struct NoAllocLayout {
    size_t status, idx, w, sorted_pair, pair_row, counts, offsets, active, n_active, max_count, act, o, total;
};

NoAllocLayout noalloc_layout(int E, int H, int I, int T, int k)
{
    NoAllocLayout L;
    const size_t P = (size_t)T * k;
    size_t off = 0;
    auto take = [&](size_t bytes) { const size_t at = off; off = align256(off + bytes); return at; };
    L.status = take(4);
    L.idx = take(4 * P);
    L.w = take(4 * P);
    L.sorted_pair = take(4 * P);
    L.pair_row = take(4 * P);
    L.counts = take(4 * (size_t)E);
    L.offsets = take(4 * ((size_t)E + 1));
    L.active = take(4 * (size_t)E);
    L.n_active = take(4);
    L.max_count = take(4);
    L.act = take(4 * P * I);
    L.o = take(4 * P * H);
    L.total = off;
    return L;
}

template <int NT, bool GU>
cudaError_t launch_canonical(const fe::CanonParams& p, int grid, int threads, cudaStream_t s)
{
    const size_t smem = fe::gemv_smem_bytes<NT>(p.K, p.TW, threads);
    fe::gemv_canonical_kernel<NT, GU><<<grid, threads, smem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

extern "C" {

fe_status fe_moe_forward_noalloc(int E, int H, int I, const uint8_t* gate_up_codes, const uint16_t* gate_up_scales,
                                 const uint8_t* down_codes, const uint16_t* down_scales, const void* x_bf16,
                                 const float* router_logits, int T, int top_k, void* y_bf16, fe_stream_t stream)
{
    if (E < 1 || E > 1024 || H <= 0 || I <= 0 || H % 32 || I % 32 || T < 0 || top_k < 1 || top_k > E)
        return FE_ERR_INVALID_ARG;
    if (T == 0) return FE_OK;
    if (!gate_up_codes || !gate_up_scales || !down_codes || !down_scales || !x_bf16 || !router_logits || !y_bf16 ||
        x_bf16 == y_bf16)
        return FE_ERR_INVALID_ARG;
    if (!aligned16(gate_up_codes) || !aligned16(gate_up_scales) || !aligned16(down_codes) || !aligned16(down_scales) ||
        (reinterpret_cast<uintptr_t>(x_bf16) & 3u) || (reinterpret_cast<uintptr_t>(y_bf16) & 3u) ||
        (reinterpret_cast<uintptr_t>(router_logits) & 3u))
        return FE_ERR_INVALID_ARG;
    const int gu_TW = pick_tile_width(H, I, true);
    const int dn_TW = pick_tile_width(I, H, false);
    if (gu_TW == 0 || dn_TW == 0) return FE_ERR_UNSUPPORTED;
    const NoAllocLayout L = noalloc_layout(E, H, I, T, top_k);
    if (L.total > kNoAllocScratchBytes) {
        snprintf(g_last_error, sizeof(g_last_error),
                 "fe_moe_forward_noalloc: T*top_k = %d pairs need %zu bytes of scratch, above the %zu-byte static "
                 "array (pairs * (I + H) * 4 bytes must stay below it)",
                 T * top_k, L.total, kNoAllocScratchBytes);
        return FE_ERR_CAPACITY;
    }
    int dev = 0;
    FE_CUDA_TRY(cudaGetDevice(&dev));
    unsigned char* scr = nullptr;
    const fe_status st0 = noalloc_setup(dev, &scr);
    if (st0 != FE_OK) return st0;
    cudaStream_t s = (cudaStream_t)stream;
    const int P = T * top_k;
    // the status word starts every call at zero (a memset node, no allocation)
    FE_CUDA_TRY(cudaMemsetAsync(scr + L.status, 0, sizeof(uint32_t), s));

    fe::RouteParams rp{};
    rp.logits = router_logits; rp.T = T; rp.E = E; rp.k = top_k;
    rp.idx = reinterpret_cast<int32_t*>(scr + L.idx);
    rp.w = reinterpret_cast<float*>(scr + L.w);
    rp.counts = reinterpret_cast<int32_t*>(scr + L.counts);
    rp.offsets = reinterpret_cast<int32_t*>(scr + L.offsets);
    rp.sorted_pair = reinterpret_cast<int32_t*>(scr + L.sorted_pair);
    rp.pair_row = reinterpret_cast<int32_t*>(scr + L.pair_row);
    rp.active = reinterpret_cast<int32_t*>(scr + L.active);
    rp.n_active = reinterpret_cast<int32_t*>(scr + L.n_active);
    rp.max_count = reinterpret_cast<int32_t*>(scr + L.max_count);
    rp.status = reinterpret_cast<uint32_t*>(scr + L.status);
    const int rthreads = std::min(fe::kRouteMaxThreads, std::max(32, roundup32(std::max(P, 32 * T))));
    fe::route_group_kernel<<<1, rthreads, fe::route_smem_bytes(E, rthreads), s>>>(rp);
    FE_CUDA_TRY(cudaGetLastError());

    const int max_active = std::min(E, P);
    fe::CanonParams cp{};
    cp.offsets = rp.offsets; cp.active = rp.active; cp.n_active = rp.n_active; cp.sorted_pair = rp.sorted_pair;
    cp.top_k = top_k;
    cp.codes = gate_up_codes; cp.scales = gate_up_scales; cp.K = H; cp.N = 2 * I; cp.TW = gu_TW;
    cp.n_tiles = I / (gu_TW / 2); cp.N_out = I; cp.x = static_cast<const uint16_t*>(x_bf16); cp.act_in = nullptr;
    cp.out = reinterpret_cast<float*>(scr + L.act);
    int threads = roundup32((gu_TW / 16) * (H / 32));
    cudaError_t e = (T == 1) ? launch_canonical<1, true>(cp, max_active * cp.n_tiles, threads, s)
                             : launch_canonical<4, true>(cp, max_active * cp.n_tiles, threads, s);
    if (e != cudaSuccess) return record_cuda(e, "noalloc gate_up launch");
    cp.codes = down_codes; cp.scales = down_scales; cp.K = I; cp.N = H; cp.TW = dn_TW; cp.n_tiles = H / dn_TW;
    cp.N_out = H; cp.x = nullptr; cp.act_in = reinterpret_cast<const float*>(scr + L.act);
    cp.out = reinterpret_cast<float*>(scr + L.o);
    threads = roundup32((dn_TW / 16) * (I / 32));
    e = (T == 1) ? launch_canonical<1, false>(cp, max_active * cp.n_tiles, threads, s)
                 : launch_canonical<4, false>(cp, max_active * cp.n_tiles, threads, s);
    if (e != cudaSuccess) return record_cuda(e, "noalloc down launch");

    dim3 cgrid((H / 8 + 255) / 256, T);
    fe::combine_kernel<false><<<cgrid, 256, 0, s>>>(reinterpret_cast<const float*>(scr + L.o), rp.w, rp.pair_row, H, top_k,
                                              static_cast<__nv_bfloat16*>(y_bf16));
    FE_CUDA_TRY(cudaGetLastError());
    return FE_OK;
}

fe_status fe_moe_noalloc_get_status(uint32_t* bits)
{
    int dev = 0;
    FE_CUDA_TRY(cudaGetDevice(&dev));
    unsigned char* scr = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_noalloc_mu);
        if (dev < 0 || dev >= 64 || !g_noalloc_dev[dev].ready) return FE_ERR_INVALID_ARG;
        scr = g_noalloc_dev[dev].scratch;
    }
    uint32_t v = 0;
    FE_CUDA_TRY(cudaDeviceSynchronize());
    FE_CUDA_TRY(cudaMemcpy(&v, scr, sizeof(v), cudaMemcpyDeviceToHost));   // the status word is at offset 0
    FE_CUDA_TRY(cudaMemset(scr, 0, sizeof(v)));
    if (bits) *bits = v;
    return v ? FE_ERR_DEVICE_STATUS : FE_OK;
}

fe_status fe_moe_noalloc_get_routing(int E, int T, int top_k, int32_t* idx, float* w, int32_t* counts,
                                     int32_t* offsets, int32_t* sorted_pair, int32_t* pair_row, fe_stream_t stream)
{
    if (E < 1 || E > 1024 || T < 0 || top_k < 1 || top_k > E) return FE_ERR_INVALID_ARG;
    int dev = 0;
    FE_CUDA_TRY(cudaGetDevice(&dev));
    unsigned char* scr = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_noalloc_mu);
        if (dev < 0 || dev >= 64 || !g_noalloc_dev[dev].ready) return FE_ERR_INVALID_ARG;
        scr = g_noalloc_dev[dev].scratch;
    }
    // the routing lists sit before act and o, at offsets that depend on E, T and top_k only
    const NoAllocLayout L = noalloc_layout(E, 64, 64, T, top_k);
    if (L.act > kNoAllocScratchBytes) return FE_ERR_CAPACITY;
    cudaStream_t s = (cudaStream_t)stream;
    const size_t P = (size_t)T * top_k;
    const cudaMemcpyKind d2d = cudaMemcpyDeviceToDevice;
    if (idx && P) FE_CUDA_TRY(cudaMemcpyAsync(idx, scr + L.idx, 4 * P, d2d, s));
    if (w && P) FE_CUDA_TRY(cudaMemcpyAsync(w, scr + L.w, 4 * P, d2d, s));
    if (counts) FE_CUDA_TRY(cudaMemcpyAsync(counts, scr + L.counts, 4 * (size_t)E, d2d, s));
    if (offsets) FE_CUDA_TRY(cudaMemcpyAsync(offsets, scr + L.offsets, 4 * ((size_t)E + 1), d2d, s));
    if (sorted_pair && P) FE_CUDA_TRY(cudaMemcpyAsync(sorted_pair, scr + L.sorted_pair, 4 * P, d2d, s));
    if (pair_row && P) FE_CUDA_TRY(cudaMemcpyAsync(pair_row, scr + L.pair_row, 4 * P, d2d, s));
    return FE_OK;
}

}  // extern "C"
