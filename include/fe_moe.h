/*
 * fe_moe: one packed FP4 mixture-of-experts FFN layer on an NVIDIA B200 (sm_100a).
 *
 * The layer is the packed MoE decode layer of the "FireEcho Engine" page
 * (sections "The Goliath Kernel: Why It's Fast" and "Speed Optimization
 * History", steps 1-5: grouped dispatch, fused gate_up projection, single-token
 * decode path, multi-expert kernel, all experts in one contiguous buffer whose
 * expert IDs are read from GPU memory), with the SiLU(gate)*up product of the
 * "FastInfer" page (section "Confirmed elementwise SwiGLU scheduling"):
 *
 *   router   per token t: the top_k experts by logit (ties to the lower expert
 *            index) in descending order are slots j = 0..top_k-1; slot weights
 *            w[t][j] = softmax over the top_k selected logits;
 *   grouping pair p = t*top_k + j goes to expert idx[t][j]; pairs are grouped
 *            by expert, ordered by pair id inside an expert;
 *   gate_up  h = x[t] . W_gu[e] (K = H, N = 2I), gate = h[0:I], up = h[I:2I],
 *            act = silu(gate) * up;
 *   down     o = act . W_dn[e] (K = I, N = H);
 *   combine  y[t] = sum_j w[t][j] * o_{t,j}, summed in slot order, rounded
 *            once to bfloat16.
 *
 * Weight format (what fe_moe_load_packed accepts): each expert matrix W[K][N]
 * is stored as 4-bit E2M1 codes (bit 3 sign, magnitudes 0, 0.5, 1, 1.5, 2, 3,
 * 4, 6; code 8 decodes to zero), two per byte with the LOW nibble holding the
 * even k, all experts in one contiguous [E][K/2][N] byte buffer, plus one
 * bfloat16 scale per group of 32 consecutive k in a [E][K/32][N] buffer:
 * W[e][k][n] = e2m1(code) * scale[e][k/32][n].  The fused gate_up matrix has
 * N = 2I columns, the gate columns [0, I) first and the up columns [I, 2I)
 * second.  Weights are dequantised in registers inside the kernels; no
 * dequantised weight is ever written to memory.
 *
 * Conventions for every entry point:
 *  - return FE_OK (0) or a negative fe_status; no exception crosses the ABI;
 *  - "device" pointers are CUDA device (or managed) memory on the handle's
 *    device, "host" pointers are ordinary host memory (pinned memory makes the
 *    copies asynchronous);
 *  - fe_stream_t is a cudaStream_t (NULL = the legacy default stream);
 *  - the library owns its weight copies and workspace; the caller owns x,
 *    logits, y and the stream; one handle must not be used on two streams at
 *    the same time;
 *  - arguments are validated on the host before anything is enqueued; an
 *    argument error enqueues nothing.
 */
#ifndef FE_MOE_H
#define FE_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct fe_moe_s* fe_moe_t;
typedef struct CUstream_st* fe_stream_t; /* the same type as cudaStream_t */

typedef enum {
    FE_OK = 0,
    FE_ERR_INVALID_ARG = -1,   /* bad dimension, null pointer, top_k out of range, ... */
    FE_ERR_UNSUPPORTED = -2,   /* valid but not supported here (group != 32, no sm_100 GPU) */
    FE_ERR_NOT_LOADED = -3,    /* forward before fe_moe_load_packed */
    FE_ERR_CAPACITY = -4,      /* T or top_k above what fe_moe_reserve reserved */
    FE_ERR_OOM = -5,           /* a device allocation failed */
    FE_ERR_CUDA = -6,          /* a CUDA runtime call failed */
    FE_ERR_DEVICE_STATUS = -7  /* a kernel flagged bad data (see fe_moe_get_status) */
} fe_status;

/* Device-side problem bits, reported through fe_moe_get_status. */
#define FE_DEVICE_BAD_EXPERT 0x1   /* an expert id outside [0, E) reached a kernel */
#define FE_DEVICE_NAN_LOGIT 0x2    /* a NaN router logit (treated as -inf) */
#define FE_DEVICE_EXCHANGE_TIMEOUT 0x4  /* single-launch decode: other CTAs' partial outputs never arrived */
#define FE_DEVICE_LOAD_TIMEOUT 0x8      /* a weight copy into shared memory never completed */
#define FE_DEVICE_TC_TIMEOUT 0x10       /* a tensor-core tile gave up waiting for its MMAs */

/* Create a handle for a layer of E experts, hidden size H and expert
 * intermediate size I on the current CUDA device.  The layer's shape is the
 * 128-expert MoE FFN of "FireEcho Engine" (section "Key Results": 30B total,
 * ~3.3B active parameters per token; "Architecture": MoEFFN, packed MoE with
 * fused dispatch); group is the number of consecutive k sharing one scale.  group must be 32; H and I
 * must be positive multiples of 32 (FE_ERR_INVALID_ARG otherwise) and of 64
 * (FE_ERR_UNSUPPORTED otherwise: the kernels read K in quads of 64); E in
 * [1, 1024].  Allocates the weight buffers (E * (H*2I + I*H) * 9/16 bytes) but
 * no workspace. */
fe_status fe_moe_create(int E, int H, int I, int group, fe_moe_t* out);

/* Allocate the forward workspace for up to max_T tokens and top_k <= max_top_k
 * ("FireEcho Engine", "Speed Optimization History" steps 6-7: buffers are
 * made once, outside the decode loop, so that the graph-captured forward
 * allocates nothing).
 * Synchronous, allocating, not capturable; call it before capturing forward in
 * a CUDA graph.  Calling it again with larger limits re-allocates. */
fe_status fe_moe_reserve(fe_moe_t h, int max_T, int max_top_k);

/* Load packed weights in the format above ("FireEcho Engine", "The Goliath
 * Kernel: Why It's Fast": all experts packed into one contiguous
 * [E, K/2, N] buffer; "Key Results": 4x compression of BF16; "Packed Marlin
 * projections": gate and up projections packed into one matrix at load
 * time).  Sizes follow from E, H, I:
 *   gate_up_codes  uint8 [E][H/2][2I],  gate_up_scales bf16 [E][H/32][2I],
 *   down_codes     uint8 [E][I/2][H],   down_scales    bf16 [E][I/32][H].
 * src_on_device = 1: the four pointers are device memory; 0: host memory.
 * The library re-lays the bytes out into its own device buffers (16-column
 * blocks in tensor-core fragment order); the caller's buffers may be freed
 * after this call returns.  Work is enqueued on stream; when I % 128 == 0 and
 * H % 256 == 0 the call then waits for the stream once, to learn whether every
 * scale allows exact f16 weights (nonzero |scale| in [2^-13, 2^13)), which the
 * tensor-core path needs. */
fe_status fe_moe_load_packed(fe_moe_t h, const uint8_t* gate_up_codes, const uint16_t* gate_up_scales,
                             const uint8_t* down_codes, const uint16_t* down_scales, int src_on_device,
                             fe_stream_t stream);

/* Load INT2 experts ("FireEcho Engine", "Quantization Formats": INT2, a
 * scalar 2-bit format, 8x, for the coldest experts; "FE-XC / INT2 Cold Expert
 * Demotion": hot experts FP4, the coldest INT2).  formats: host uint8 [E], 1 =
 * expert e runs on the INT2 weights given here, 0 = on its E2M1 weights of
 * fe_moe_load_packed (which stays required: it makes the layer loaded; the
 * E2M1 bytes of INT2 experts are then ignored).  INT2 format: a 2-bit code q
 * stands for (q - 1.5) times the bf16 scale of its group of 32 along K
 * (scale = bf16(max|w| / 1.5), as fe_moe_pack_int2_host makes them); four
 * codes per byte, the code of k = 4b + i in bits 2i, 2i+1 of byte row b:
 *   gate_up_codes uint8 [E][H/4][2I], gate_up_scales bf16 [E][H/32][2I],
 *   down_codes    uint8 [E][I/4][H],  down_scales    bf16 [E][I/32][H],
 * full size (rows of E2M1 experts are ignored), host (src_on_device = 0) or
 * device memory.  The first call allocates the INT2 buffers (15 * E * I * H
 * / 16 bytes); the call waits for stream.  A layer with INT2 experts runs on the single-launch decode path
 * only (T <= 8, T * top_k <= 16): fe_moe_forward returns FE_ERR_UNSUPPORTED
 * for larger T, and a stack of such layers makes one launch per layer.
 * H % 64 and I % 64 must be 0 (else FE_ERR_UNSUPPORTED). */
/* Block-scaled FP4 variant of the projections ("FireEcho Engine", "The Goliath
 * Kernel: Why It's Fast": FP4 codes at the matmul; the tensor cores' FP4 rate
 * takes only E4M3 scale factors per 16 elements, which the bf16 group scales
 * are not).  Re-encodes the layer's packed weights -- the same arrays, layout
 * and src_on_device convention as fe_moe_load_packed -- into NVFP4, per output
 * column along K:
 *   g = amax / 2688 (fp32 row scale), s_b = E4M3(amax_b / (6 g)) per block of
 *   16 (nearest, ties to even, at most 448), code = E2M1(w / (s_b g)) (nearest,
 *   ties to even), every step in fp32,
 * into tile images the kernels copy as they are (27 E I H / 16 bytes with
 * their scale factors, plus the row scales; allocated by the first call).  With FE_PATH_NVFP4 set, fe_moe_forward then encodes x per token and
 * act (bf16) per pair row the same way and runs both projections as
 * kind::mxf4nvf4 MMAs with fp32 accumulation: an approximation of the layer,
 * whose distance to it the caller measures (it is not within the layer's
 * tolerance).  Needs H % 256 == 0 and I % 256 == 0 (else FE_ERR_UNSUPPORTED)
 * and fe_moe_load_packed for the routing workspace's layer; token images are
 * workspace of fe_moe_reserve (tile slots x max(H, I) / 256 x 36 KiB).  Work is
 * enqueued on stream; host sources are staged through a stream-ordered buffer.
 * On this path fe_moe_forward also needs x 16-byte aligned (else
 * FE_ERR_INVALID_ARG). */
fe_status fe_moe_load_nvfp4(fe_moe_t h, const uint8_t* gate_up_codes, const uint16_t* gate_up_scales,
                            const uint8_t* down_codes, const uint16_t* down_scales, int src_on_device,
                            fe_stream_t stream);

/* The NVFP4 row encoding of fe_moe_load_nvfp4 on rows of fp32 values: src
 * device float [rows][K] -> device codes uint8 [rows][K/2] (two per byte, the
 * low nibble for the even k; bit 3 the sign), E4M3 scale factors uint8
 * [rows][K/16], row scales float [rows].  A value decodes as E2M1(code) *
 * E4M3(scale factor) * row scale.  K % 16 == 0, K >= 16, src 16-byte and
 * codes 8-byte aligned (else FE_ERR_INVALID_ARG).  Asynchronous on stream. */
fe_status fe_moe_nvfp4_quantize_device(const float* src, int64_t rows, int64_t K, uint8_t* codes, uint8_t* sf,
                                       float* row_scale, fe_stream_t stream);

fe_status fe_moe_load_int2(fe_moe_t h, const uint8_t* formats, const uint8_t* gate_up_codes,
                           const uint16_t* gate_up_scales, const uint8_t* down_codes, const uint16_t* down_scales,
                           int src_on_device, fe_stream_t stream);

/* The layer: y = MoE(x) ("FireEcho Engine", "Speed Optimization History"
 * steps 1-5 and "The Goliath Kernel: Why It's Fast": grouped dispatch with
 * expert ids read from device memory, fused gate_up projection, FP4 decoded
 * inside the matmul loop; "FastInfer", "Confirmed elementwise SwiGLU
 * scheduling": SiLU(gate) * up).  x_bf16 device bf16 [T][H], router_logits device
 * float [T][E], y_bf16 device bf16 [T][H] (must not alias x).  T = 0 is a
 * no-op.  1 <= top_k <= min(E, max_top_k), T <= max_T.  Asynchronous on
 * stream: no host synchronisation and no allocation, so it can be captured in
 * a CUDA graph and replayed with new contents in the same buffers.  The
 * routing (idx, w, grouping) stays in the workspace until the next call. */
fe_status fe_moe_forward(fe_moe_t h, const void* x_bf16, const float* router_logits, int T, int top_k,
                         void* y_bf16, fe_stream_t stream);

/* The router GEMM fused with the top-k ("FireEcho Engine", "Architecture":
 * MoEFFN, the packed MoE whose dispatch starts from the router's scores;
 * "Speed Optimization History" step 1: the router in front of the grouped
 * dispatch, expert ids chosen on the GPU).  In one launch:
 *   logits[t][e] = sum_h x[t][h] * W_r[e][h]   (bf16 products, fp32 sums),
 * then per token the top_k experts by logit (ties to the lower index) and the
 * softmax of their logits, as fe_moe_forward routes.
 *   x_bf16        device bf16 [T][H], 16-byte aligned (caller-owned, read);
 *   w_router_bf16 device bf16 [E][H], one row per expert, 16-byte aligned;
 *   logits        device float [T][E] (written);
 *   idx, w        device int32 / float [T][top_k] in slot order (written), or
 *                 NULL to skip.
 * The sums run in fp32 in an order of the library's choosing (deterministic
 * for given T, H, E): within sum_h |x W_r| * H * 2^-24 of the exact sum.  Needs
 * H % 64 == 0, E <= 512, top_k <= 32 and top_k * ceil(E/32 rounded up to a
 * power of two) <= 256 (else FE_ERR_UNSUPPORTED), T <= max_T (else
 * FE_ERR_CAPACITY); misaligned or NULL required pointers: FE_ERR_INVALID_ARG.
 * T = 0 is a no-op.  Asynchronous on stream, no allocation: capturable. */
fe_status fe_moe_router(fe_moe_t h, const void* x_bf16, const void* w_router_bf16, int T, int top_k,
                        float* logits, int32_t* idx, float* w, fe_stream_t stream);

/* The layer from x alone: fe_moe_router (logits into the caller's `logits`,
 * device float [T][E], which the call also returns), then fe_moe_forward on
 * those logits.  Same argument rules as both; the layer's own routing (idx,
 * w, grouping) is the router's, taken again from the same fp32 logits.
 * Asynchronous on stream, no allocation. */
fe_status fe_moe_forward_router(fe_moe_t h, const void* x_bf16, const void* w_router_bf16, int T, int top_k,
                                void* y_bf16, float* logits, fe_stream_t stream);

/* The layer on HOST buffers (no counterpart on the pages: the same layer as
 * fe_moe_forward for a caller whose x and logits are in host memory): copies
 * x and the logits to the device, runs
 * fe_moe_forward and copies y back, then waits for the stream.  Same argument
 * rules as fe_moe_forward (T <= max_T).  Synchronous. */
fe_status fe_moe_forward_host(fe_moe_t h, const uint16_t* x_bf16_host, const float* router_logits_host, int T,
                              int top_k, uint16_t* y_bf16_host, fe_stream_t stream);

/* Copy the routing of the last forward into caller device buffers (any may
 * be NULL) -- the router and grouping of "FireEcho Engine", "Speed
 * Optimization History" step 1 (grouped dispatch) and "The Goliath Kernel:
 * Why It's Fast" (expert ids stay on the GPU): idx int32 [T][top_k], w float [T][top_k], offsets int32 [E+1]
 * (exclusive scan of the per-expert pair counts), sorted_pair int32
 * [T*top_k] (pair ids ordered by (expert, pair id)).  Enqueued on stream. */
fe_status fe_moe_get_routing(fe_moe_t h, int32_t* idx, float* w, int32_t* offsets, int32_t* sorted_pair,
                             fe_stream_t stream);

/* Copy the rest of the last forward's grouping into caller device buffers
 * (either may be NULL): counts int32 [E] (pairs per expert) and pair_row
 * int32 [T*top_k] (pair_row[p] = the grouped position of pair p, the inverse
 * of sorted_pair, which the ordered combine reads).  Enqueued on stream. */
fe_status fe_moe_get_grouping(fe_moe_t h, int32_t* counts, int32_t* pair_row, fe_stream_t stream);

/* Wait for the device and return FE_ERR_DEVICE_STATUS if a kernel flagged a
 * problem since the last call (the bits go to *bits if non-NULL), FE_OK
 * otherwise; clears the flags. */
fe_status fe_moe_get_status(fe_moe_t h, uint32_t* bits);

/* Compute paths of fe_moe_forward. */
#define FE_PATH_AUTO 0          /* chosen per call from T, top_k and the shape */
#define FE_PATH_GEMV 1          /* routing + grouped mma.sync gate_up and down + combine (any T): persistent
                                   streaming kernels, or one CTA per unit when their ring does not fit */
#define FE_PATH_TCGEN05 2       /* routing + tcgen05 tensor-core tiles + combine (large T; I % 128 == 0,
                                   H % 256 == 0, scales in the exact-f16 range) */
#define FE_PATH_FUSED_DECODE 3  /* one kernel for the whole layer (T <= 8, T * top_k <= 16), its CTAs all
                                   resident at once (checked from the occupancy; otherwise not taken) */
#define FE_PATH_NVFP4 4         /* routing + block-scaled FP4 tensor-core tiles (tcgen05.mma kind::mxf4nvf4)
                                   + combine: an approximation of the layer (fe_moe_load_nvfp4); any T;
                                   never chosen by FE_PATH_AUTO */

/* Force a compute path (FE_PATH_*; any other value: FE_ERR_INVALID_ARG);
 * FE_ERR_UNSUPPORTED from forward if the forced path cannot run the call.
 * A stack whose layers have a forced path runs one layer at a time on it.
 * For tests and measurements (and to choose the FE_PATH_NVFP4 variant). */
fe_status fe_moe_set_path(fe_moe_t h, int path);

/* Which path the last successful forward took and how many kernels it
 * enqueued. */
fe_status fe_moe_last_forward_info(fe_moe_t h, int* path, int* kernels);

/* Diagnostics: when device_buf (device memory, [number of SMs][64] uint64)
 * is set, every CTA of the single-launch decode kernel writes stamps of its
 * phases there: slot i (0..31) holds %globaltimer in ns and slot 32 + i the
 * SM's clock64 at the same point (0 start, 8 previous grid done, 10 routed,
 * 9 grouped, 1 copies issued, 2 x staged, 11 / 13 first / last unit's
 * gate_up bytes landed, 3 units done, 26 every CTA arrived (CTAs that sum an
 * output slice), 5 end).  Slots a CTA does not reach keep their old
 * contents.  The streaming kernels of the moderate-T path write
 * [2][number of SMs][8] instead (gate_up, then down; per CTA clock64 at
 * start, range known, first unit landed, end; its unit count; %globaltimer
 * at start and end).  The persistent stack launch (fe_moe_stack_forward at
 * T = 1) uses the buffer of its first layer's handle as [number of SMs][16]:
 * per CTA, compute thread 0's clock64 cycles summed over the stack per phase
 * (0 x wait, 1 gate_up bytes wait, 2 gate_up, 3 SwiGLU step, 4 down bytes
 * wait, 5 down, 6 slot release, 7 partial-buffer guard, 8 partial stores),
 * 9 its units, 10 the whole layer loop, and the exchange warp's 11 poll
 * cycles, 12 polls, 13 slice-sum cycles, 14 of them landing the words, 15
 * adding them.  NULL switches it off. */
fe_status fe_moe_set_trace(fe_moe_t h, unsigned long long* device_buf);

/* For tests of the failure path: with unreachable = 1 the single-launch
 * decode kernel's CTAs that sum an output slice wait for one arrival more than
 * the launch has (it never comes) for at most wait_ns nanoseconds, then set
 * FE_DEVICE_EXCHANGE_TIMEOUT and leave their slice of y unwritten; every wait
 * on the CTA's own copies keeps its full bound, so no copy is in flight when a
 * CTA returns.  unreachable = 0 restores the normal wait (bounded at 200 ms).
 * No counterpart on the pages. */
fe_status fe_moe_set_exchange_test(fe_moe_t h, int unreachable, unsigned long long wait_ns);

/* Human-readable text of a status code (static storage). */
const char* fe_moe_status_string(fe_status s);

/* Free every buffer of the handle.  Waits for the device first. */
void fe_moe_destroy(fe_moe_t h);

/* The load-time packer: float W [E][K][N] -> E2M1 codes [E][K/2][N] and bf16
 * scales [E][K/32][N].  Per group of 32 along k and column n: scale =
 * bf16_rne(max|w| / 6) (the division in float32); code = the E2M1 value
 * nearest to w / scale (float32 division), exact midpoints to the value with
 * an even mantissa bit, ratios beyond 6 clamped to 6, a zero magnitude stored
 * as code 0, an all-zero group as scale 0 and codes 0.  K % 32 == 0.
 * Host version: host pointers, multithreaded, synchronous. */
fe_status fe_moe_pack_host(const float* W, int64_t E, int64_t K, int64_t N, uint8_t* codes, uint16_t* scales);

/* The same packer on the GPU: device pointers, enqueued on stream.  Produces
 * bytes identical to fe_moe_pack_host. */
fe_status fe_moe_pack_device(const float* W, int64_t E, int64_t K, int64_t N, uint8_t* codes, uint16_t* scales,
                             fe_stream_t stream);

/* The INT2 packer of fe_moe_load_int2's format: float W [E][K][N] -> codes
 * [E][K/4][N] and bf16 scales [E][K/32][N].  Per group of 32 along k and
 * column n: scale = bf16_rne(max|w| / 1.5) (float32 division); the code q of
 * r = w / scale (float32) is the nearest of the levels q - 1.5, an exact
 * midpoint (r = -1, 0, 1) going to the level above; an all-zero group stores
 * scale 0 and codes 2.  K % 32 == 0.  Host version: host pointers,
 * multithreaded, synchronous. */
fe_status fe_moe_pack_int2_host(const float* W, int64_t E, int64_t K, int64_t N, uint8_t* codes, uint16_t* scales);

/* The same INT2 packer on the GPU: device pointers, enqueued on stream; bytes
 * identical to fe_moe_pack_int2_host. */
fe_status fe_moe_pack_int2_device(const float* W, int64_t E, int64_t K, int64_t N, uint8_t* codes,
                                  uint16_t* scales, fe_stream_t stream);

/* Allocation-free forward.  No counterpart on the source pages: an addition for
 * callers that must not allocate device memory -- for instance code running
 * under an external memory manager that owns every device byte, or code that
 * may not call cudaMalloc, a stream-ordered pool or any allocating library
 * routine at the point where it runs the layer.  It needs no handle and no
 * workspace: the caller passes the packed weights in the format of
 * fe_moe_load_packed (device memory, 16-byte aligned, read in place), x, the
 * logits and y; the routing lists and intermediate activations live in one
 * static device array of 4 MiB that every GPU which loads the library holds
 * until the process exits.  Calls whose T * top_k * (I + H) * 4 bytes plus a
 * few KiB of routing lists exceed that array return FE_ERR_CAPACITY with the
 * reason in fe_moe_last_error(); nothing is enqueued then.  The first call on
 * each device, with that device current, looks up the array's device address
 * and sets kernel attributes (neither allocates); make that first call before
 * any stream capture.  Every call shares the array and leaves its contents
 * behind: each call clears the array's status word when it starts (an
 * asynchronous memset on the stream, which allocates nothing) and writes
 * every other scratch word before it reads it, but calls whose kernels
 * overlap on the GPU (other streams, other threads) race on the array and
 * must be serialised by the caller.  Same sizes and layouts as fe_moe_create
 * + fe_moe_forward; no allocation, no host synchronisation; argument errors
 * as fe_moe_forward.  Device-side problems (a NaN logit, an expert id out of
 * range) are reported by fe_moe_noalloc_get_status, not fe_moe_get_status. */
fe_status fe_moe_forward_noalloc(int E, int H, int I, const uint8_t* gate_up_codes, const uint16_t* gate_up_scales,
                                 const uint8_t* down_codes, const uint16_t* down_scales, const void* x_bf16,
                                 const float* router_logits, int T, int top_k, void* y_bf16, fe_stream_t stream);

/* Device-side problem bits (FE_DEVICE_BAD_EXPERT, FE_DEVICE_NAN_LOGIT) of the
 * last fe_moe_forward_noalloc call on the current device.  Waits for the
 * device, returns FE_ERR_DEVICE_STATUS if a bit is set (the bits go to *bits
 * if non-NULL) and FE_OK otherwise, and clears the word.  The word is shared
 * by every call on the device, like the rest of the array.  Allocates
 * nothing; FE_ERR_INVALID_ARG before the first fe_moe_forward_noalloc call on
 * the device. */
fe_status fe_moe_noalloc_get_status(uint32_t* bits);

/* Copy the routing and grouping of the last fe_moe_forward_noalloc call on
 * the current device (which must have had these E, T and top_k) from the
 * static array into caller device buffers, any of which may be NULL: idx int32
 * [T][top_k], w float [T][top_k], counts int32 [E], offsets int32 [E+1],
 * sorted_pair and pair_row int32 [T*top_k] (as fe_moe_get_routing and
 * fe_moe_get_grouping).  Enqueued on stream; allocates nothing. */
fe_status fe_moe_noalloc_get_routing(int E, int T, int top_k, int32_t* idx, float* w, int32_t* counts,
                                     int32_t* offsets, int32_t* sorted_pair, int32_t* pair_row, fe_stream_t stream);

/* ---- a stack of layers -------------------------------------------------------
 * n layers run back to back on one stream, as in the 48-layer graph-captured
 * decode forward of "FireEcho Engine" (section "Benchmark Results", row L6,
 * and "Speed Optimization History" step 7). */
typedef struct fe_moe_stack_s* fe_moe_stack_t;

/* Build a stack over n_layers >= 1 handles, which it does not own (they must
 * outlive the stack and keep the reservation they had when it was made; a
 * layer reserved again afterwards makes the stack fall back to one launch per
 * layer): all on one device, with the same E and H, each reserved and
 * loaded.  Allocates staging for fe_moe_stack_forward_host: x and y of
 * every layer ([n_layers (+1)][max_T][H] bf16, max_T the smallest
 * reservation among the layers) and the logits of every layer. */
fe_status fe_moe_stack_create(const fe_moe_t* layers, int n_layers, fe_moe_stack_t* out);

/* Layer l = 0 .. n_layers-1, in order on stream: y_l = layer[l](x_l) with
 * x_l = x_bf16 + l*T*H, logits_l = logits + l*T*E and y_l = y_bf16 + l*T*H
 * (device memory; bf16 [T][H], float [T][E]).  y_l must not overlap x_l.
 * Passing y_bf16 = x_bf16 + T*H chains the layers (layer l + 1 reads what
 * layer l wrote, stream order making it safe); separate buffers make them
 * independent.  Each layer runs as fe_moe_forward on its own handle; every
 * layer's arguments are checked before the first launch.  Asynchronous, no
 * allocation, no host synchronisation: capturable in one CUDA graph. */
fe_status fe_moe_stack_forward(fe_moe_stack_t s, const void* x_bf16, const float* logits, int T, int top_k,
                               void* y_bf16, fe_stream_t stream);

/* The stack on HOST buffers: copies the inputs and the logits of every layer
 * [n_layers][T][E] to the device (one copy each), runs fe_moe_stack_forward,
 * copies the outputs back and waits for the stream.  chained = 0: x
 * [n_layers][T][H] in, y [n_layers][T][H] out (independent layers); chained
 * = 1: x [T][H] is layer 0's input, each layer feeds the next, y [T][H] is the
 * last layer's output.  Synchronous. */
fe_status fe_moe_stack_forward_host(fe_moe_stack_t s, const uint16_t* x_bf16_host, const float* logits_host, int T,
                                    int top_k, uint16_t* y_bf16_host, int chained, fe_stream_t stream);

/* Cross-layer streaming on (1, the default) or off (0).  On: a call at T = 1
 * whose layers all take the single-launch decode kernel (same shape, x and y
 * chained as y = x + T*H or not overlapping) runs the whole stack as ONE
 * persistent launch, one CTA per SM; a call at T <= 4 tokens whose routing is
 * sparse (4 * T * top_k <= E, so the tokens rarely share an expert) runs as
 * one such launch per token, token t's rows of every layer in launch t (the
 * first launch also writes every layer's routing and grouping of all T
 * tokens, as fe_moe_forward leaves them): every layer is routed up front (the stack
 * takes every layer's logits at once), each CTA streams its share of the
 * layers' weights through a ring of shared-memory slots without stopping at
 * layer boundaries, so the next layer's weights arrive while the current one
 * finishes ("FireEcho Engine", "Benchmark Results": row L2, the next layer
 * fetched ahead of use, and row L6, the 48-layer forward as one graph).
 * Device-side problems of that launch are reported through the first layer's
 * handle (fe_moe_get_status).  Off, or any other call: one fe_moe_forward per
 * layer.  Both are bit-reproducible run to run; they differ from each other in
 * how the per-CTA partial outputs are grouped before the fixed-order sum, so
 * their outputs agree to within rounding, not bit for bit. */
fe_status fe_moe_stack_set_prefetch(fe_moe_stack_t s, int on);

/* Kernels the last fe_moe_stack_forward enqueued (1 per token for the
 * persistent launches); -1 for a NULL stack. */
int fe_moe_stack_last_launches(fe_moe_stack_t s);

/* Free the stack's buffers (not the layers).  Waits for the device first. */
void fe_moe_stack_destroy(fe_moe_stack_t s);

/* Text of the last CUDA failure behind an FE_ERR_CUDA / FE_ERR_OOM returned to
 * this thread ("" if none); static thread-local storage. */
const char* fe_moe_last_error(void);

/* Bytes of device memory the handle holds (weights + workspace). */
size_t fe_moe_device_bytes(fe_moe_t h);

#ifdef __cplusplus
}
#endif

#endif /* FE_MOE_H */
