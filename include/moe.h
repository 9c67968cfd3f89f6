/*
 * moe.h -- C ABI of libmoe.so: the forward pass of a routed Mixture-of-Experts FFN layer on
 * one NVIDIA B200 (sm_100a), for decode (a few tokens) and prefill (thousands of tokens).
 *
 * The layer (as the colibri README and the iliria page describe it, sections "The idea" and
 * "What's implemented", and the Glacial page, section "What works"):
 *
 *   1. router: logits[t][e] = sum_i x[t][i] * Wr[e][i]; then either
 *        softmax top-k (Granite style): the k largest logits, weights = softmax over those k;
 *        sigmoid + selection bias (DeepSeek-V3 style, "noaux_tc", routed_scaling_factor):
 *        key = sigmoid(logit) + bias[e] picks the k experts, the weights are
 *        routed_scaling_factor * sigmoid / (sum of the chosen sigmoids) -- the bias is used
 *        for selection only;
 *      equal keys go to the lower expert index; the k outputs of a token are in rank order.
 *   2. batch-union dispatch: every chosen expert's weights are read once and applied to every
 *      token routed to it ("Batch-union MoE", colibri README).
 *   3. SwiGLU experts: g = Wg x, u = Wu x, h = silu(g) * u, y = Wd h, over packed int4 weights
 *      with one fp32 scale per output row dequantised on use ("Quantization kernels ... packed
 *      int4 ... per-row scales ... dequant-on-use", colibri README), or over bf16 weights.
 *   4. combine: out[t] = sum over the chosen experts (ascending expert index) of
 *      weight * y, plus the shared expert with weight 1 ("shared expert", colibri README).
 *
 * Conventions used by every entry point:
 *   - Pointers marked "device" must point to memory of the CUDA device that was current when
 *     the layer was created (or, for moe_pack_int4, the current device); "host" means CPU
 *     memory (pageable or pinned).
 *   - bf16 data are passed as uint16_t bit patterns.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL is the legacy default stream).  Only
 *     the calls documented as synchronous wait for the device.
 *   - No C++ exception or CUDA error escapes: every failure is a moe_status.  Argument errors
 *     are returned before anything is enqueued.  moe_route, moe_forward and moe_route_noalloc
 *     first clear an error that an earlier, unrelated runtime call left pending (the CUDA
 *     runtime's last-error state), so that they report only their own launches.  Errors found
 *     by the device while running (a bounded wait that ran out, a value out of range) are
 *     latched in the layer's device status word and returned by moe_last_error().
 *   - The library never allocates on the hot path: moe_route / moe_forward use the workspace
 *     that moe_layer_create allocated for `max_tokens` tokens.
 */
#ifndef QEFFN_MOE_H
#define QEFFN_MOE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct moe_layer moe_layer;          /* opaque */
typedef struct CUstream_st *moe_stream;      /* the same type as cudaStream_t */

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,   /* a NULL pointer, a size out of range, a misaligned pointer */
    MOE_ERR_CUDA = 2,          /* a CUDA runtime call failed (launch, copy, allocation flags) */
    MOE_ERR_OOM = 3,           /* workspace allocation failed */
    MOE_ERR_TIMEOUT = 4,       /* a bounded device-side wait gave up */
    MOE_ERR_RANGE = 5,         /* non-finite weights given to the packer; an fp16 overflow of h */
    MOE_ERR_UNSUPPORTED = 6    /* a shape this build has no kernel for */
} moe_status;

enum { MOE_ROUTER_SOFTMAX_TOPK = 0, MOE_ROUTER_SIGMOID_BIAS = 1 };
/* Weight containers (colibri README, "What's implemented": int8 / packed int4 / packed int2
 * quantisation with per-row scales, dequant-on-use): packed int4 (two codes per byte), bf16,
 * int8 (one code of the 8-bit tier per byte), packed int2 (four codes of the 2-bit tier per
 * byte).  The int8 and int2 containers run on the general decode kernels at every batch size;
 * the single-launch decode path and the tcgen05 grouped GEMMs take packed int4. */
enum { MOE_W_INT4_ROWSCALE = 0, MOE_W_BF16 = 1, MOE_W_INT8_ROWSCALE = 2, MOE_W_INT2_ROWSCALE = 3 };

typedef struct {
    int32_t d;                   /* hidden size; even, and a multiple of 64 */
    int32_t f;                   /* routed expert intermediate size; a multiple of 64 */
    int32_t n_experts;           /* E, 1..1024 */
    int32_t top_k;               /* k, 1..min(E, 32) */
    int32_t n_shared;            /* 0 or 1 */
    int32_t f_shared;            /* shared expert intermediate size (multiple of 64); ignored if n_shared == 0 */
    int32_t max_tokens;          /* largest T that moe_route / moe_forward accept (>= 1) */
    int32_t router;              /* MOE_ROUTER_* */
    float routed_scaling_factor; /* multiplies the renormalised weights (1.0 for the softmax router) */
    int32_t wkind;               /* MOE_W_* */
    int32_t out_bf16;            /* 0: moe_forward writes fp32 [T][d]; 1: bf16 [T][d] */
} moe_config;

/*
 * Expert weights, all device pointers, all borrowed: the caller keeps them alive and
 * unchanged for the life of the layer.  Row-major throughout; one expert's data are
 * contiguous.  The fused gate/up matrix holds the f gate rows first, then the f up rows (the
 * split-at-the-row-boundary convention of the open-1b-verify page, "Tensor mapping").
 *
 *   int4 (MOE_W_INT4_ROWSCALE): the output of moe_pack_int4 --
 *     gate_up        [E][2f][d/2] bytes     gate_up_scale [E][2f] fp32
 *     down           [E][d][f/2]  bytes     down_scale    [E][d]  fp32
 *   bf16 (MOE_W_BF16): gate_up [E][2f][d], down [E][d][f]; the scale pointers are ignored.
 *   int8 (MOE_W_INT8_ROWSCALE): the output of moe_pack_int8 -- gate_up [E][2f][d] int8,
 *     down [E][d][f] int8, scales as for int4.
 *   int2 (MOE_W_INT2_ROWSCALE): the output of moe_pack_int2 -- gate_up [E][2f][d/4] bytes,
 *     down [E][d][f/4] bytes, scales as for int4.
 *   shared_*: the same for the single shared expert (with f_shared in place of f), or NULL
 *   when n_shared == 0.
 *   router_w [E][d] fp32; router_bias [E] fp32 for the sigmoid router (NULL means zeros).
 * Every pointer must be 16-byte aligned.
 */
typedef struct {
    const float *router_w;
    const float *router_bias;
    const void *gate_up;
    const float *gate_up_scale;
    const void *down;
    const float *down_scale;
    const void *shared_gate_up;
    const float *shared_gate_up_scale;
    const void *shared_down;
    const float *shared_down_scale;
} moe_weights;

/*
 * moe_pack_int4 -- quantise an fp32 matrix to the packed int4 container (colibri README,
 * "What's implemented": packed int4 with per-row scales, validated bit-identical to the int8
 * container).  For each row: scale = fp32(max|w| / 7); q = clamp(round-half-even(fp32(w /
 * scale)), -8, 7); a row of zeros has scale 0 and codes 0.  Byte j of a row holds column 2j in
 * its low nibble and column 2j+1 in its high nibble, each a 4-bit two's-complement code.
 *
 *   w       device, [rows][cols] fp32
 *   packed  device, [rows][cols/2] bytes (written)
 *   scales  device, [rows] fp32 (written)
 *   rows >= 0; cols even and > 0.
 * Synchronous: waits for `stream`, because it reports non-finite input (MOE_ERR_RANGE; such
 * elements are written as code 0) -- it is a set-up call, not part of the forward pass.
 */
moe_status moe_pack_int4(const float *w, int64_t rows, int64_t cols, uint8_t *packed, float *scales,
                         moe_stream stream);

/*
 * moe_pack_int8 / moe_pack_int2 -- the 8-bit and 2-bit tiers of the same per-row rule (colibri
 * README, "What's implemented": int8 / packed int4 / packed int2 quantisation, per-row scales):
 * qmax = 2^(b-1) - 1 (127 or 1); scale = fp32(max|w| / qmax); q = clamp(round-half-even(fp32(w /
 * scale)), -qmax - 1, qmax); a row of zeros has scale 0 and codes 0.
 *   moe_pack_int8: q device [rows][cols] int8, one code per byte; cols > 0.
 *   moe_pack_int2: packed device [rows][cols/4] bytes, column 4j + i of a row in bits 2i .. 2i+1 of
 *                  byte j (a 2-bit two's-complement code); cols a multiple of 4.
 *   w device [rows][cols] fp32; scales device [rows] fp32 (written).  Errors and synchronisation
 *   as for moe_pack_int4 (non-finite input: MOE_ERR_RANGE, its codes written as 0).
 */
moe_status moe_pack_int8(const float *w, int64_t rows, int64_t cols, int8_t *q, float *scales, moe_stream stream);
moe_status moe_pack_int2(const float *w, int64_t rows, int64_t cols, uint8_t *packed, float *scales,
                         moe_stream stream);

/*
 * moe_layer_create -- validate the configuration, borrow the weights, and allocate the
 * workspace for cfg->max_tokens tokens on the current CUDA device.  *out is set only on
 * success.  Errors: MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_OOM, MOE_ERR_CUDA.
 */
moe_status moe_layer_create(const moe_config *cfg, const moe_weights *w, moe_layer **out);

/*
 * moe_route -- router and top-k only (step 1 above).
 *   x    device, [T][d] bf16
 *   idx  device, [T][k] int32 (written): chosen experts in rank order (-1 where adaptive top-p,
 *        MOE_OPT_ROUTER_TOP_P, dropped one)
 *   w    device, [T][k] fp32 (written): their gate weights (computed in fp64, rounded once; 0 for
 *        a dropped expert)
 *   0 <= T <= max_tokens.  Asynchronous.  The logits are accumulated in fp64.
 */
moe_status moe_route(moe_layer *layer, const uint16_t *x, int32_t T, int32_t *idx, float *w,
                     moe_stream stream);

/*
 * moe_forward -- the whole layer, steps 1 to 4.
 *   x    device, [T][d] bf16
 *   out  device, [T][d] fp32, or bf16 when cfg->out_bf16 (written)
 *   0 <= T <= max_tokens.  Asynchronous: no host synchronisation and no allocation.  Calls on
 *   one layer must not overlap on the device (they share its workspace).
 */
moe_status moe_forward(moe_layer *layer, const uint16_t *x, int32_t T, void *out, moe_stream stream);

/*
 * moe_layer_set_expert -- point routed expert e (0 <= e < E) at weights anywhere in device memory:
 * a ragged table of experts in place of one contiguous [E] array (iliria page, "What's
 * implemented": grouped MoE over a ragged descriptor of expert slabs; colibri README, "The idea":
 * experts streamed on demand).  gate_up, gate_up_scale, down, down_scale: device pointers in
 * the layer's container format for ONE expert ([2f][...] rows, [2f] scales, [d][...] rows, [d]
 * scales; the scale pointers are ignored for bf16 weights), 16-byte aligned, borrowed like the
 * layer's other weights.  Asynchronous: the layer's device pointer table is updated on `stream`,
 * in order with the forwards enqueued on that stream (order calls on other streams yourself).
 * Once any expert has been re-pointed the tcgen05 grouped-GEMM path, whose tensor maps cover the
 * contiguous arrays, is no longer used (MOE_OPT_PREFILL_AVAILABLE reads 0); every other path
 * reads the table.  Errors: MOE_ERR_INVALID_ARG (index, NULL or misaligned pointer),
 * MOE_ERR_CUDA.
 */
moe_status moe_layer_set_expert(moe_layer *layer, int32_t e, const void *gate_up, const float *gate_up_scale,
                                const void *down, const float *down_scale, moe_stream stream);

/*
 * moe_forward_host -- moe_forward on host buffers: copies x host->device, runs the layer,
 * brings out back to the host, and waits for `stream`.  x_host [T][d] bf16; out_host [T][d]
 * fp32 or bf16.  Synchronous.  x goes through one of two staging areas inside the workspace.
 * An output of at most 1 MiB in pinned (mapped) host memory is written there by the layer's
 * last kernel directly; any other output goes through a staging area and one device->host
 * copy.
 */
moe_status moe_forward_host(moe_layer *layer, const uint16_t *x_host, int32_t T, void *out_host,
                            moe_stream stream);

/*
 * moe_forward_host_async -- moe_forward_host without the final wait: the layer and the return
 * of out are enqueued on `stream` and the call returns.  The host->device copy of x runs on a
 * copy stream of the layer's own, into the staging area the call before last used, so that it
 * can overlap the previous call's kernels; `stream` waits for it before the layer runs.  Calls
 * on one stream may follow each other at once.  x_host must stay unchanged until the stream has
 * passed the call (an event or a synchronize), and out_host holds the result only from then
 * on.  With pinned buffers the copies are asynchronous to the host; with pageable ones the
 * runtime may wait inside the call.  Asynchronous.
 */
moe_status moe_forward_host_async(moe_layer *layer, const uint16_t *x_host, int32_t T, void *out_host,
                                  moe_stream stream);

/*
 * moe_last_error -- wait for the layer's most recent stream, then return (and clear) the
 * device status word: MOE_OK, MOE_ERR_TIMEOUT or MOE_ERR_RANGE; MOE_ERR_CUDA if the wait
 * itself failed.  Synchronous.
 */
moe_status moe_last_error(moe_layer *layer);

/* moe_layer_destroy -- free the workspace (after waiting for the layer's last stream).  NULL is
 * ignored.  The borrowed weights are not touched. */
void moe_layer_destroy(moe_layer *layer);

/*
 * Layer options.
 *   MOE_OPT_PREFILL_MIN_TOKENS  batches with T >= value run the experts as tcgen05 grouped GEMMs
 *                               (when the shape allows: int4 weights, d, f and f_shared multiples
 *                               of 128); smaller batches use the HBM-streaming decode kernels.
 *                               Default 128; value >= 1.  Both paths give the same results within
 *                               the layer's tolerance.
 *   MOE_OPT_PREFILL_AVAILABLE   (read only) 1 if this layer has the grouped-GEMM path.
 * Setting an option is host-only and takes effect at the next moe_forward.
 */
/*   MOE_OPT_SINGLE_TOKEN_KERNELS how a T = 1 batch runs when the shape allows (int4 weights, d a
 *                               multiple of 1024 up to 8192, f_shared == f, k + shared <= 10):
 *                               2 (default where f is 1024 or 2048 and E <= 256): the whole layer
 *                               in one cooperative launch (router, top-k, gate/up, down, combine);
 *                               1: the fused router launch, then the single-token gate/up and
 *                               down+combine kernels; 0: the general decode kernels.  A request
 *                               for a mode the shape does not allow falls back to the next lower
 *                               one; get returns the mode in use.  Same results within tolerance.
 *                               Mode 2 is a cooperative launch of one CTA per SM: it starts when
 *                               every SM can take its CTA, so kernels of other streams running at
 *                               the same time delay it.  In mode 2 a T = 2 batch with int4
 *                               weights and ceil(d / SMs) <= 48 (and 16 warps' rings in shared
 *                               memory where E > 224) also runs as one launch: each shared-expert
 *                               row is read once for both tokens; mode 1 or 0 sends T = 2 to the
 *                               batch kernels.  Such a launch does not write MOE_DEBUG_ULIST.
 */
/*   MOE_OPT_PROGRAMMATIC_LAUNCH  1 (default): chained kernels (the single-token kernels, and the
 *                               batch expert kernels and combine after the router) start early
 *                               with programmatic dependent launch and wait on the device for
 *                               their inputs; 0: ordinary stream order.  Same results.
 */
/*   MOE_OPT_WAIT_LIMIT_US        time limit, in microseconds (100 .. 10,000,000; default 2,000,000), of
 *                               every bounded device-side wait of the grouped-GEMM kernels.  When a
 *                               wait runs out, the kernel latches MOE_ERR_TIMEOUT, lets the copies it
 *                               issued land, frees its tensor memory and returns; moe_last_error
 *                               reports it and the layer stays usable.  (The decode kernels keep a
 *                               fixed 2 s limit.)
 *   MOE_OPT_TEST_SKIP_GEMM_B_COPIES  test hook for that error path: 1 makes the grouped-GEMM kernels'
 *                               activation-tile producer issue no copies, so the MMA warp's wait for
 *                               them runs out after MOE_OPT_WAIT_LIMIT_US and the forward reports
 *                               MOE_ERR_TIMEOUT (its output is then undefined); 0 (default) is normal
 *                               operation.  Nothing faults or hangs: every waiter gives up within the
 *                               limit.
 */
/*   MOE_OPT_ROUTER_GROUPS        group-limited selection (colibri README, "What's implemented": the
 *                               DeepSeek-V3 router's noaux_tc): value = n_group + 65536 * topk_group.
 *                               The E experts form n_group contiguous groups of E / n_group; a group's
 *                               score is the sum of its two largest selection keys; only the
 *                               topk_group best groups (equal scores: the lower group first) stay
 *                               selectable, and the top-k runs over their experts.  Gate weights as
 *                               without groups.  n_group = 1 (default) is the plain router;
 *                               otherwise n_group <= 32, E % n_group == 0, 1 <= topk_group <= n_group
 *                               and topk_group * E / n_group >= k.
 *   MOE_OPT_ROUTER_TOP_P         adaptive expert top-p (colibri README, "Quick start": --topp), in
 *                               millionths (0 .. 1,000,000; 0 and 1,000,000 = off, the default).  Of
 *                               a token's k chosen experts, the shortest rank-order prefix whose gate
 *                               weights reach p of the k weights' total is kept and rescaled to that
 *                               total; the others are dropped: moe_route writes index -1 and weight
 *                               0 for them, and moe_forward never reads their weights.
 *   While either variant is on, T = 1 batches run on the general decode kernels (the single-token
 *   paths take the plain router only).  moe_route_noalloc always uses the plain router.
 *   MOE_OPT_UNION_TENSOR_CORES   batches of 2 .. prefill-threshold tokens with int4 experts (d, f and
 *                               the shared f multiples of 1024): 1 (default) runs gate/up and down as
 *                               tensor-core products of 16 weight rows by up to 8 tokens; 0 runs the
 *                               general kernels (FP32-pipe dot products).  Results agree within the
 *                               layer's tolerance, not bit for bit.
 *   MOE_OPT_PHASE_TRACE          1: the single launch records the phase times that MOE_DEBUG_TRACE
 *                               returns; 0 (default): it records none (each stamp is a timer read
 *                               on the path of the CTA's first thread).  Same results.
 */
enum { MOE_OPT_PREFILL_MIN_TOKENS = 0, MOE_OPT_PREFILL_AVAILABLE = 1, MOE_OPT_SINGLE_TOKEN_KERNELS = 2,
       MOE_OPT_PROGRAMMATIC_LAUNCH = 3, MOE_OPT_WAIT_LIMIT_US = 4, MOE_OPT_TEST_SKIP_GEMM_B_COPIES = 5,
       MOE_OPT_ROUTER_GROUPS = 6, MOE_OPT_ROUTER_TOP_P = 7, MOE_OPT_UNION_TENSOR_CORES = 8,
       MOE_OPT_PHASE_TRACE = 9 };
moe_status moe_layer_set_option(moe_layer *layer, int32_t option, int64_t value);
moe_status moe_layer_get_option(const moe_layer *layer, int32_t option, int64_t *value);

/*
 * moe_layer_debug_read -- copy one intermediate of the most recent moe_forward to host memory
 * (waits for the layer's last stream).  For tests and debugging; the contents depend on which
 * kernels ran (see each item).  `bytes` is the size of `dst`; at most the item's size is copied.
 *   MOE_DEBUG_H      h = silu(g) * u, fp16 [slots][fmax] (slot = routed slot, then T*k + t for the
 *                    shared expert; K order of the grouped-GEMM path is permuted in groups of 8;
 *                    the single-launch path (T = 1 or 2) has rows [T*(k+1)][f], routed slot
 *                    t*k + rank, and stores 8-value chunk c of a row at position
 *                    (c % (f/256)) * 32 + c / (f/256))
 *   MOE_DEBUG_Y      y per slot, fp32 [slots][d] (not written by the single-token kernels)
 *   MOE_DEBUG_IDX / MOE_DEBUG_W / MOE_DEBUG_ASC   int32 / fp32 / int32 [T][k]
 *   MOE_DEBUG_ULIST  int32 [E] unique chosen experts, ascending;  MOE_DEBUG_CNT int32 [E]
 *                    (CNT is not written by the single-launch path, ULIST not by it at T = 2)
 *   MOE_DEBUG_XSUM   fp64 [T]
 *   MOE_DEBUG_TRACE  uint64 [SMs][16]: for the single-launch path with MOE_OPT_PHASE_TRACE on, the
 *                    %globaltimer value (ns) at which each CTA passed its phase boundaries: 0 start,
 *                    11 x in shared memory, 1 router pieces stored, 2 arrived at the first grid
 *                    barrier, 3 x rearranged and the shared rows done, 4 first grid barrier passed,
 *                    5 router pieces gathered, 12 candidates, 13 ranks and pointers, 14 and 15
 *                    around a proxy fence, 6 experts selected, 7 routed gate/up done, 8 h
 *                    complete, 9 down done, 10 output stored.  A call that runs the
 *                    small-batch router (2 <= T <= 32, or T = 1 off the single launch) writes
 *                    one row per router block instead (block z * groups + g): 0 start, 1 x and
 *                    the router slice staged, 2 partial logits stored, 3 past the group's
 *                    counter, 4 the group's logits stored, 5 past the last counter, then in
 *                    the last block 6 selection done, 7 counted, 8 offsets, 9 slots placed
 */
enum { MOE_DEBUG_H = 0, MOE_DEBUG_Y = 1, MOE_DEBUG_IDX = 2, MOE_DEBUG_W = 3, MOE_DEBUG_ASC = 4,
       MOE_DEBUG_ULIST = 5, MOE_DEBUG_CNT = 6, MOE_DEBUG_XSUM = 7, MOE_DEBUG_TRACE = 8 };
moe_status moe_layer_debug_read(moe_layer *layer, int32_t item, void *dst, int64_t bytes);

/* Bytes of device workspace the layer holds. */
int64_t moe_layer_workspace_bytes(const moe_layer *layer);

/* Number of kernel launches the most recent moe_forward / moe_route enqueued (host bookkeeping). */
int32_t moe_layer_last_launches(const moe_layer *layer);

/* Static text for a status code. */
const char *moe_status_str(moe_status status);

/*
 * Per-kernel timing.  While enabled, every kernel launch of the layer is bracketed by a pair of
 * CUDA events recorded on the launching stream; moe_profile_read waits for the layer's last
 * stream and returns (and resets) the summed device time and the launch count of one kernel.
 * Off by default; turning it on adds two event records per launch.
 */
enum {
    MOE_KERNEL_ROUTER_LOGITS = 0,   /* router GEMV, fp64 accumulation */
    MOE_KERNEL_TOPK = 1,            /* top-k selection and gate weights */
    MOE_KERNEL_BUCKET = 2,          /* histogram, scan, scatter, unique list */
    MOE_KERNEL_GATEUP = 3,          /* decode: gate/up rows + SiLU */
    MOE_KERNEL_DOWN = 4,            /* decode: down rows */
    MOE_KERNEL_COMBINE = 5,         /* weighted combine with the shared expert */
    MOE_KERNEL_GATHER = 6,          /* prefill: x rows gathered per expert */
    MOE_KERNEL_GEMM_GATEUP = 7,     /* prefill: tcgen05 grouped GEMM gate/up + SiLU */
    MOE_KERNEL_GEMM_DOWN = 8,       /* prefill: tcgen05 grouped GEMM down */
    MOE_KERNEL_FUSED = 9,           /* decode, T = 1: the whole layer in one cooperative launch */
    MOE_KERNEL_COUNT = 10
};
/*
 * moe_route_noalloc -- the routing step of moe_route, for callers that must not allocate device
 * memory and so cannot create a layer: code running while a CUDA graph is captured (an
 * allocation call breaks the capture), engines that serve every device byte from their own
 * preallocated arena, and real-time loops that allow no allocation after start-up.  The pages
 * have no counterpart: this is a deployment convenience of this library.
 *
 *   cfg       only d, n_experts, top_k, router and routed_scaling_factor are read
 *   router_w  device, [E][d] fp32;  router_bias  device, [E] fp32 or NULL (sigmoid router)
 *   x         device, [T][d] bf16;  idx [T][k] int32 and w [T][k] fp32 are written (device)
 * The only scratch is a fixed 1 MiB array inside libmoe.so's device image, present on every GPU
 * that loads the library until the process exits.  A call needs T*E*8 (rounded up to 256) +
 * T*8 bytes of it; a larger request returns MOE_ERR_UNSUPPORTED (E = 256 allows T <= 510).
 * The first call on each device looks up that array's device address and sets the router
 * kernel's shared-memory limit (neither allocates); make that first call before any stream
 * capture.  The address is looked up once per device and kept until the process exits: it is
 * not looked up again, so after cudaDeviceReset() on a device this entry point must not be
 * called on that device again.  Every call on a device shares the array and the array keeps the last call's
 * contents (each call overwrites all it reads); calls that overlap on the GPU -- on different
 * streams, or from different host threads -- race on it.  Asynchronous; no allocation, no
 * synchronisation.
 */
moe_status moe_route_noalloc(const moe_config *cfg, const float *router_w, const float *router_bias,
                             const uint16_t *x, int32_t T, int32_t *idx, float *w, moe_stream stream);

/*
 * A device-memory tier of routed experts in front of host memory (colibri README, "The idea":
 * routed experts streamed on demand behind a per-layer LRU cache and an optional pinned hot set;
 * iliria page, "What's implemented": pinned/LRU slabs behind a ragged descriptor).  n_slots
 * expert-sized device buffers hold the experts in use; host memory holds all E.
 *
 * moe_expert_cache_create -- cfg as for moe_layer_create.  device: router_w, router_bias and the
 *   shared expert (device pointers, borrowed); its routed-expert fields are ignored.  host: the
 *   routed experts in host memory (the same fields and layouts as moe_weights; pinned memory
 *   makes the copies asynchronous), borrowed.  1 <= n_slots <= E.  Allocates the slots
 *   (n_slots x one expert's bytes) and creates the layer (moe_expert_cache_layer), whose experts
 *   are read through its pointer table.  Synchronous.
 * moe_expert_cache_prepare -- route x ([T][d] bf16, device; 0 <= T <= max_tokens) and make every
 *   expert it routes to resident: a free slot, else the least recently used slot whose expert is
 *   neither pinned nor needed by this batch, is filled by host-to-device copies on `stream`, and
 *   the layer's table is pointed at it.  Waits for the routing (the host needs the expert ids);
 *   the copies stay asynchronous.  Call moe_forward on the same stream afterwards.
 *   MOE_ERR_UNSUPPORTED: the batch needs more experts than the free and evictable slots.
 * moe_expert_cache_pin -- pinned = 1 keeps expert e resident once loaded (the hot tier); 0 unpins.
 * moe_expert_cache_stats -- experts found resident (hits), copied in (misses), bytes copied in,
 *   and slots in use.  moe_expert_cache_slot_of -- the slot holding expert e, or -1.
 * moe_expert_cache_destroy -- waits for the layer's last stream, frees the slots and the layer.
 */
typedef struct moe_expert_cache moe_expert_cache;
moe_status moe_expert_cache_create(const moe_config *cfg, const moe_weights *device, const moe_weights *host,
                                   int32_t n_slots, moe_expert_cache **out);
moe_layer *moe_expert_cache_layer(moe_expert_cache *cache);
moe_status moe_expert_cache_prepare(moe_expert_cache *cache, const uint16_t *x, int32_t T, moe_stream stream);
moe_status moe_expert_cache_pin(moe_expert_cache *cache, int32_t e, int32_t pinned);
moe_status moe_expert_cache_stats(const moe_expert_cache *cache, int64_t *hits, int64_t *misses, int64_t *bytes_in,
                                  int32_t *resident);
int32_t moe_expert_cache_slot_of(const moe_expert_cache *cache, int32_t e);
void moe_expert_cache_destroy(moe_expert_cache *cache);

moe_status moe_profile_enable(moe_layer *layer, int32_t on);
moe_status moe_profile_read(moe_layer *layer, int32_t kernel, double *total_ms, int64_t *launches);
const char *moe_kernel_name(int32_t kernel);

#ifdef __cplusplus
}
#endif
#endif /* QEFFN_MOE_H */
