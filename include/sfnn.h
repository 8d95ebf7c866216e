/*
 * sfnn.h -- activation-sparse FFN decode on NVIDIA B200 (sm_100a): the C ABI.
 *
 * The operation.  For one FFN layer with n neurons over model width d,
 *
 *     y = sum_{i in S(x)} act_i(x) * W_down[:, i]
 *     ReLU : act_i(x) = relu(W_up[i] . x + b_i)
 *     ReGLU: act_i(x) = relu(W_gate[i] . x + b_i) * (W_up[i] . x)
 *     S(x) = { i : sigmoid(relu(x . A) . B + c)_i > 0.5 } = { i : (relu(x.A).B + c)_i > 0 }
 *
 * and the rows of W_up / W_gate and the columns of W_down that belong to
 * neurons outside S(x) are neither read nor multiplied.  Sources: ReLU makes
 * most FFN neurons inactive, an inactive neuron's down-projection row adds an
 * exact zero and can be skipped, turning the step into a sparse-vector times
 * dense-matrix product that saves both bytes and FLOPs (53ai.com "sparsity for
 * LLM inference" page, section 激活稀疏, activation sparsity); a small per-layer
 * MLP predicts which MLP neurons will be active and only those are computed
 * (same page, sections 概述 and 自适应稀疏预测器, the PowerInfer overview and
 * its adaptive sparse predictor; DejaVu's MLP predictor in section 如何推理加速);
 * the predictor used here is a rank-r two-layer MLP, sigmoid(relu(x.A).B + c),
 * thresholded at 0.5, evaluated as z > 0 because sigmoid is strictly
 * increasing with sigmoid(0) = 1/2 (a tie z == 0 and a NaN are inactive).
 * Neurons are stored in descending order of an offline activation frequency
 * ("hot" neurons first), after PowerInfer's offline hot/cold profiling (same
 * page, section 概述; hexiedandong.com PowerInfer news page, the power-law
 * paragraph on figure (a)).
 *
 * Conventions for every entry point.
 *  - Pointers are DEVICE pointers unless a parameter says "host".  The caller
 *    owns every buffer it passes; a handle owns the layer's re-laid-out weights
 *    and its scratch memory.
 *  - Element type: x / X and all weights use the handle's wdtype (IEEE fp32
 *    or fp16); outputs y / Y are fp32; index lists and counts are int32.
 *    x / X must start on a 16-byte boundary (SFNN_ERR_INVALID_ARG otherwise):
 *    they are read with 16-byte vector loads and bulk async copies.
 *  - Every call after sfnn_create is asynchronous on `stream` and never
 *    synchronises the host, never aborts and never throws.  Argument errors
 *    are returned at once and launch nothing.  Errors found on the device
 *    (an out-of-range index passed in, a bounded wait that ran out) are
 *    latched in the handle and returned by sfnn_get_error.
 *  - A handle must not be used from two streams at the same time: its scratch
 *    memory is shared by its calls.
 *  - The fused kernels (single token, few tokens, look-ahead stack) run one CTA per
 *    SM that fills the SM's registers, and synchronise all their CTAs with grid
 *    barriers: every SM must be able to take one of them.  A kernel that occupies an
 *    SM on another stream delays the CTA bound for it, and the barriers wait for that
 *    CTA (correct, but slower); if it does not arrive within about one second the
 *    launch gives up and latches SFNN_ERR_TIMEOUT.  Two fused launches of different
 *    handles on concurrent streams can each hold part of the SMs and so time out:
 *    serialise them.
 *  - Index lists have set semantics: they hold each selected neuron once, in
 *    the caller's original numbering, in the handle's internal (hotness) order,
 *    which is deterministic.
 *  - Deterministic results: the same inputs give bitwise the same outputs.
 */
#ifndef SFNN_H
#define SFNN_H

#include <stdint.h>

/* Entry points are the only symbols the shared library exports. */
#if defined(__GNUC__)
#define SFNN_API __attribute__((visibility("default")))
#else
#define SFNN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t (struct CUstream_st *); 0 is the legacy default stream. */
typedef struct CUstream_st *sfnn_stream_t;
/* Same type as cudaEvent_t (struct CUevent_st *). */
typedef struct CUevent_st *sfnn_event_t;

typedef struct sfnn_ctx *sfnn_handle;

typedef enum {
    SFNN_OK = 0,
    SFNN_ERR_INVALID_ARG = 1, /* a null pointer, a size out of range, an inconsistent descriptor */
    SFNN_ERR_CUDA = 2,        /* a CUDA runtime call or kernel launch failed */
    SFNN_ERR_OOM = 3,         /* device memory allocation failed in sfnn_create */
    SFNN_ERR_UNSUPPORTED = 4, /* valid but outside what this build handles (see sfnn_create) */
    SFNN_ERR_TIMEOUT = 5      /* a bounded device-side wait gave up (latched) */
} sfnn_status;

typedef enum { SFNN_RELU = 0, SFNN_REGLU = 1 } sfnn_act;
typedef enum { SFNN_F32 = 0, SFNN_F16 = 1, SFNN_I8 = 2, SFNN_I4 = 3 } sfnn_dtype;

/*
 * Which kernels the batched path (b > 1, and explicit sets) uses.  The tensor-core
 * path runs the batch's predictor (hidden layer and logits as dense GEMMs; h enters
 * the logits as an fp16 hi + lo pair, about 22 significant bits) and the union's
 * up/gate and down projections (gathered GEMMs) on tcgen05 tensor cores, with fp32
 * accumulation and the activations rounded to fp16 between the two projections; it
 * needs fp16 weights, d a multiple of 128 and max_batch >= 2 (the predictor part also
 * r a multiple of 64, else the CUDA-core predictor runs).  The fused path runs a batch
 * of 2 to 4 tokens in one launch of the multi-token kernel on CUDA cores (the
 * single-token kernel's plan with every weight read once for all tokens: predictor
 * rows, and the union of the tokens' active rows, each row applied only to the tokens
 * whose sets hold it); it needs fp16 weights, d <= 16384 and r <= 1024.  AUTO takes the
 * fused path for 2 to 4 tokens and the tensor cores for more: a union of a few tokens'
 * sets is too thin to be a real contraction, while from 8 tokens on it is dense enough
 * that the tensor cores' gathered GEMMs beat CUDA cores; where a path does not fit a
 * layer, the next one serves (fused -> tensor cores -> CUDA cores).
 */
typedef enum {
    SFNN_BATCH_AUTO = 0,
    SFNN_BATCH_CUDA_CORE = 1,   /* multi-token gather on CUDA cores */
    SFNN_BATCH_TENSOR_CORE = 2, /* dense and gathered GEMMs on tcgen05 tensor cores */
    SFNN_BATCH_FUSED = 3        /* 2..4 tokens: one fused launch on CUDA cores; more: as AUTO */
} sfnn_batch_path;

/*
 * One FFN layer in PyTorch layouts (row-major):
 *   w_up   [n x d]  up.weight                (device, wdtype)
 *   w_gate [n x d]  gate.weight, ReGLU only; NULL for ReLU
 *   b      [n]      bias of the ReLU'd projection (up for ReLU, gate for ReGLU)
 *   w_down [d x n]  down.weight
 *   pa     [d x r]  predictor A;  pb [r x n] predictor B;  pc [n] predictor bias c
 *   hotness[n]      HOST, optional: offline activation frequency of each neuron;
 *                   NULL keeps the original order.  NaN counts as lowest.
 * The inputs are read during sfnn_create only; they may be freed once it returns.
 */
typedef struct {
    int32_t d, n, r;   /* d <= 65536, n <= 2^20 (else SFNN_ERR_UNSUPPORTED) */
    int32_t max_batch; /* largest b later passed to sfnn_forward_batch / sfnn_forward_stack, 1..32 */
    int32_t act;       /* sfnn_act */
    int32_t wdtype;    /* sfnn_dtype */
    const void *w_up;
    const void *w_gate;
    const void *b;
    const void *w_down;
    const void *pa;
    const void *pb;
    const void *pc;
    const float *hotness;
    /*
     * Storage of the FFN rows (w_up, w_gate, w_down), given in wdtype as usual:
     * SFNN_I8 / SFNN_I4 store them as int8 / int4 codes with one fp32 scale per neuron
     * and projection (weight-only quantization; the predictor, b, x and all arithmetic
     * keep their types).  The rule, in IEEE fp32, with qmax = 127 (int8) or 7 (int4):
     * scale = max|w| / qmax over the neuron's row (its column of w_down), code = w / scale
     * rounded to nearest even, clamped to +-qmax; an all-zero row has scale 0.  int4
     * codes are packed two per byte, element 2k in the low nibble of byte k.  Needs
     * wdtype = SFNN_F16 and d a multiple of 16 (int8) or 32 (int4); such a layer runs
     * the fused single-token path only (sfnn_forward without explicit sets,
     * sfnn_forward_batch and sfnn_forward_stack[_lookahead] with b = 1) and sfnn_predict;
     * other calls return SFNN_ERR_UNSUPPORTED.  Any other value (0 included) stores the rows in wdtype.
     * The pages deploy weight-quantized models (PowerInfer in INT4 on the smaller PC,
     * 53ai.com "sparsity for LLM inference" page, evaluation) without fixing a scheme.
     */
    int32_t rows_dtype;
    /*
     * Storage order of the neurons when a hotness profile is given (sfnn_order):
     * SFNN_ORDER_DEALT (0, the default) deals the hotness ranks round-robin to the SM
     * tiles of the fused kernels, hottest first inside each tile, so every tile gets the
     * same mix of hot and cold neurons; SFNN_ORDER_PACKED (1) stores the neurons in
     * plain descending hotness, the hot ones contiguous at the front (one tile then holds
     * the hottest neurons; the few-token path reads no hot prefix).  Both follow
     * PowerInfer's offline hot/cold profiling (53ai.com page, section 概述).
     */
    int32_t order;
} sfnn_layer_desc;

typedef enum { SFNN_ORDER_DEALT = 0, SFNN_ORDER_PACKED = 1 } sfnn_order;

/* Read-only facts about a handle (sizes in bytes). */
typedef struct {
    int32_t d, n, r, max_batch, act, wdtype;
    int32_t num_sms;              /* SMs of the device the handle lives on */
    int32_t batch_path;           /* sfnn_batch_path in force */
    int64_t weight_bytes;         /* re-laid-out weights held by the handle */
    int64_t scratch_bytes;        /* scratch memory held by the handle */
    int64_t predictor_bytes;      /* bytes of A, B and c one token's predictor reads */
    int64_t row_bytes_per_neuron; /* bytes of rows + bias one active neuron costs */
    int64_t launches;             /* kernels launched (or captured) by this handle so far */
} sfnn_info;

/*
 * Build a handle for one layer on the current device.  Re-lays the weights out
 * for the decode path: neurons in descending hotness; each neuron's rows
 * (gate, up, and its W_down column as a contiguous row) stored together;
 * A transposed to [r x d]; B transposed to neuron-major [n x r].
 * Requirements: d, n, r >= 1; d and r multiples of 8 (fp16) or 4 (fp32);
 * 1 <= max_batch <= 32; r * max_batch <= 32768; int8 rows: fp16 weights, d a
 * multiple of 16 and a layer the fused kernel fits (SFNN_ERR_UNSUPPORTED otherwise).
 * Allocates device memory (SFNN_ERR_OOM) and synchronises `stream` before
 * returning.  On error *out is set to NULL.
 */
SFNN_API sfnn_status sfnn_create(const sfnn_layer_desc *desc, sfnn_stream_t stream, sfnn_handle *out);

/* Free a handle (synchronises its device).  NULL is accepted. */
SFNN_API sfnn_status sfnn_destroy(sfnn_handle h);

/*
 * Predictor only: the set S(x) for one token.
 *   x     [d] wdtype
 *   idx   [n] int32 out: the |S| selected neurons first (caller numbering); capacity n
 *   count [1] int32 out: |S|
 */
SFNN_API sfnn_status sfnn_predict(sfnn_handle h, const void *x, int32_t *idx, int32_t *count, sfnn_stream_t stream);

/*
 * One decode step for one token: y = sum_{i in S} act_i(x) W_down[:, i].
 *   x     [d] wdtype
 *   idx   NULL: S = S(x) from the predictor.  Otherwise [*count] int32 neuron
 *         indices (caller numbering) that replace the predictor's set; order is
 *         free, duplicates count once, out-of-range entries are skipped and
 *         latch SFNN_ERR_INVALID_ARG.
 *   count [1] int32 (device), read only when idx != NULL; clamped to [0, n]
 *   y     [d] fp32 out
 */
SFNN_API sfnn_status sfnn_forward(sfnn_handle h, const void *x, const int32_t *idx, const int32_t *count, float *y,
                         sfnn_stream_t stream);

/*
 * b independent tokens at once (1 <= b <= max_batch): row t of Y equals
 * sfnn_forward of X[t] (within rounding: the tensor-core path rounds the
 * activations to fp16).  The union of the b predicted sets is read once and
 * applied to the tokens active on each row: as a batch's sets accumulate, the
 * benefit of sparsity shrinks (53ai.com page, section 工程效果), so the rows are
 * shared by every token that needs them.  The kernels follow sfnn_set_batch_path.
 * With b = 1 the fused single-token kernel runs (as in sfnn_forward, unless it is
 * disabled), and idx/counts return the set that kernel itself decided and read:
 * each tile's active positions as its rows were gathered, listed by one small
 * kernel after it.  A layer with quantized rows returns SFNN_ERR_UNSUPPORTED for b > 1.
 *   X      [b x d] wdtype;  Y [b x d] fp32 out
 *   idx    [b x n] int32 out or NULL: token t's set in row t (first counts[t] entries)
 *   counts [b] int32 out or NULL: |S_t|
 */
SFNN_API sfnn_status sfnn_forward_batch(sfnn_handle h, const void *X, int32_t b, float *Y, int32_t *idx, int32_t *counts,
                               sfnn_stream_t stream);

/*
 * A stack of layers with a residual stream:  X_{l+1} = X_l + FFN_l(round(X_l)),
 * where round() converts the fp32 residual to the layers' wdtype (nearest even).
 * The pages name no normalisation between the layers; none is applied.  With
 * b = 1 every layer runs the fused single-token kernel (unless disabled), and
 * idx/counts, when requested, return the sets those launches used; with b > 1, the
 * batched path.
 * All layers share d, wdtype and max_batch >= b (and n when idx != NULL).
 *   layers [num_layers] HOST array of handles
 *   X0     [b x d] fp32 in;  XL [b x d] fp32 out (may alias X0)
 *   idx    [num_layers x b x n] int32 out or NULL;  counts [num_layers x b] int32 out or NULL
 */
SFNN_API sfnn_status sfnn_forward_stack(const sfnn_handle *layers, int32_t num_layers, const float *X0, int32_t b,
                               float *XL, int32_t *idx, int32_t *counts, sfnn_stream_t stream);

/*
 * The same residual stack with every layer's active set predicted one layer ahead:
 * layer l+1's predictor (its own A, B, c) takes layer l's input round(X_l), so it can
 * run beside layer l instead of in front of layer l+1 -- DejaVu's asynchronous
 * predictor, which forecasts the next layer's sparsity one step early (53ai.com
 * "sparsity for LLM inference" page, section "如何推理加速").  Layer 0 predicts from
 * round(X_0).  The sets, and so XL, may differ from sfnn_forward_stack's.
 * With b = 1, and every layer on the fused kernel with the same number of tiles
 * (SMs), the stack runs as num_layers + 1 launches of one look-ahead kernel: launch l
 * does layer l's rows on the set launch l-1 predicted and layer l+1's predictor, with
 * one bounded grid barrier; idx/counts, when requested, return the lists each launch
 * consumed (listed after it by one small kernel; with sets requested, one handle
 * serving two consecutive layers takes the batched path instead, whose lists it
 * would otherwise overwrite).  Otherwise the batched path, with each layer's
 * prediction issued before the previous layer's reduce.
 * Arguments, sharing rules and idx/counts layout as sfnn_forward_stack.
 */
SFNN_API sfnn_status sfnn_forward_stack_lookahead(const sfnn_handle *layers, int32_t num_layers, const float *X0,
                                         int32_t b, float *XL, int32_t *idx, int32_t *counts, sfnn_stream_t stream);

/*
 * Enable (default) or disable the fused single-token kernel, which runs a whole
 * decode step of one token in one launch: one persistent CTA per SM owning a tile of
 * neurons, the predictor's rows and the active neurons' rows streamed through
 * shared memory, two grid-wide barriers with bounded waits.  Disabled, one token runs
 * through the same multi-kernel path as a batch.  SFNN_ERR_UNSUPPORTED when enabling
 * it on a layer it does not fit (shared memory or SM count).
 */
SFNN_API sfnn_status sfnn_set_fused_decode(sfnn_handle h, int32_t enable);

/*
 * The single-token fused kernel's rebalancing of active rows over its CTAs: each CTA keeps
 * the first `quota` active rows of its own tile, and the rows past the quota in all tiles
 * are shared out evenly over the CTAs after a grid barrier (results within rounding of
 * quota 0, and deterministic for a given quota).  By default the quota is 0.8 of a tile's
 * expected active count under the hotness profile when that count is 20 or more, else 0
 * (no rebalancing).  quota >= 0 sets it (clamped to a tile's size); -1 restores the
 * default.  Takes effect at the next launch.
 */
SFNN_API sfnn_status sfnn_set_fused_quota(sfnn_handle h, int32_t quota);

/*
 * The few-token fused kernel's rebalancing of union rows over its CTAs (on by default when
 * the hotness profile makes it pay, as the single-token kernel's).  With it, the CTA that
 * sums a row into its partial depends on the other tokens' sets, so a token's y can differ
 * in rounding with the batch it is in (still deterministic for a given batch); enable = 0
 * switches it off, and each token's y then does not depend on the other tokens at all.
 * Takes effect at the next launch.
 */
SFNN_API sfnn_status sfnn_set_batch_quota(sfnn_handle h, int32_t enable);

/*
 * The tensor-core batch path's kernel shapes (a tuning knob; the results do not depend on
 * it beyond the order in which partial sums are added).  Up projection: up_ctas_per_sm =
 * its CTAs per SM (1 or 2, capped by how many fit in shared memory; the union's (128-row
 * tile, K step) pairs are shared out evenly among them), up_chunks_per_step = 64-wide K
 * chunks of every row staged per step (1 or 2; two make each row's reads 256 contiguous
 * bytes).  Down projection: down_tiles_per_cta = 128-column output tiles per CTA (1 or 2;
 * two make each W_down row's reads 512 contiguous bytes; needs d a multiple of 256, else
 * 1 is used).  Defaults 2, 2, 2.  -1 keeps a value.  SFNN_ERR_INVALID_ARG outside those
 * sets; SFNN_ERR_UNSUPPORTED when the layer has no tensor-core batch path.  Takes effect at
 * the next launch.
 */
SFNN_API sfnn_status sfnn_set_batch_tc_shape(sfnn_handle h, int32_t up_ctas_per_sm, int32_t up_chunks_per_step,
                                             int32_t down_tiles_per_cta);

/*
 * Measures, on this handle, which path serves AUTO batches of multi_max + 1 .. 2 multi_max
 * tokens faster (multi_max: the few-token kernel's largest batch, 4 when it fits; at most
 * the handle's max_batch): two few-token launches of at most multi_max tokens each, or the
 * tensor-core batch path, on synthetic unit-variance tokens (fixed seed), 3 warm-up and 10
 * timed calls each (the tensor-core path twice, around the other), and makes AUTO take the
 * two launches for each such b where they are at least 5 % faster (SFNN_BATCH_FUSED always
 * takes them).  Without this call AUTO takes the tensor-core path there.  ms_out (null, or
 * 2 (2 multi_max + 1) floats) receives per b the milliseconds of one call of each path, at
 * [2b] (two launches) and [2b + 1] (tensor cores).
 * Allocates and frees temporary device memory and synchronises `stream`: a set-up call, not
 * for graph capture.  SFNN_OK with nothing measured when the handle has no such b.
 */
SFNN_API sfnn_status sfnn_tune_batch_paths(sfnn_handle h, float *ms_out, sfnn_stream_t stream);

/*
 * The few-token fused kernel's request depths, as sfnn_set_fused_depths (the results do not
 * depend on them): bstages = B^T half rows staged per warp (2, 4, 6 or 8), c2pre = W_down
 * rows requested while the up/gate rows stream (0 to 8), c1depth = up/gate segments in
 * flight per warp (1 or 2), c2stages = W_down rows in flight (1, 2, 4 or 8, capped by the
 * staging region: 8 when a W_down row is at most 8 KB, else 4).  -1 keeps a value.
 * SFNN_ERR_INVALID_ARG outside those sets; SFNN_ERR_UNSUPPORTED (nothing changed) when the
 * kernel's shared memory would not fit or the handle has no few-token kernel.
 */
SFNN_API sfnn_status sfnn_set_batch_depths(sfnn_handle h, int32_t bstages, int32_t c2pre, int32_t c1depth,
                                           int32_t c2stages);

/*
 * The single-token fused kernel's request depths (a tuning knob; the results do not depend
 * on them): bstages = B^T rows staged per warp in phase B (1, 2, 3, 4, 6 or 8), c2pre =
 * W_down rows requested while the up/gate rows stream (0 to 16), c1depth = up/gate segments
 * in flight per warp (1 or 2), c2stages = W_down rows in flight in the down phase (1, 2, 4,
 * 8 or 16, capped by the kernel's staging region: 16 when a W_down row is at most 8 KB,
 * 8 up to 16 KB, else 4).  -1 keeps a value.  SFNN_ERR_INVALID_ARG for a value outside those sets;
 * SFNN_ERR_UNSUPPORTED (nothing changed) when the kernel's shared memory would not fit or
 * the layer has no fused kernel.  Takes effect at the next launch.
 */
SFNN_API sfnn_status sfnn_set_fused_depths(sfnn_handle h, int32_t bstages, int32_t c2pre, int32_t c1depth,
                                           int32_t c2stages);

/*
 * The fused few-token path (SFNN_BATCH_FUSED, and AUTO for 2 to 4 tokens) reads the
 * hot prefix of the layer densely (enabled by default): the neurons that the offline
 * hotness profile puts in a b-token batch's union with probability >= 0.99
 * (1 - (1 - p)^b >= 0.99, at most 64 per SM tile) have their gate/up rows read and
 * multiplied for every token while the predictor's grid barrier completes, before the
 * sets are known; the cold tail is gathered by the union as usual.  The rows of a
 * prefix neuron that no token's set holds are read and dropped (the set semantics are
 * unchanged: a row applies only to the tokens whose sets hold it, and y is bitwise the
 * same either way).  This is the power-law split of the pages -- a few hot neurons
 * carry most activations (hexiedandong.com PowerInfer news page, the paragraph on
 * figure (a)) and every token of a batch needs them (53ai.com page, section 工程效果).
 * Without a hotness profile there is no prefix.  Disabling it keeps every read sparse.
 */
SFNN_API sfnn_status sfnn_set_hot_prefix(sfnn_handle h, int32_t enable);

/*
 * Fault injection for tests (synchronises `stream`): the next fused decode launch
 * of h finds its grid barrier unable to complete, waits out its bound (about one
 * second), returns without a result and latches SFNN_ERR_TIMEOUT; sfnn_get_error
 * reports it and restores the barrier, after which h works normally.
 */
SFNN_API sfnn_status sfnn_debug_stall_next_barrier(sfnn_handle h, sfnn_stream_t stream);

/* Choose the batched path (sfnn_batch_path); SFNN_BATCH_AUTO by default.
 * SFNN_ERR_UNSUPPORTED for SFNN_BATCH_TENSOR_CORE on a layer that path cannot serve. */
SFNN_API sfnn_status sfnn_set_batch_path(sfnn_handle h, int32_t path);

/*
 * Diagnostics: when `before`/`after` are non-NULL, the next sfnn_forward or
 * sfnn_forward_batch call of this handle records `before` on its stream just
 * before the first kernel of its hot path and `after` just after the last one;
 * the pair is consumed by that call.  Events may be recorded while the stream
 * is being captured into a CUDA graph.
 */
SFNN_API sfnn_status sfnn_set_profile_events(sfnn_handle h, sfnn_event_t before, sfnn_event_t after);

/*
 * The predictor for one token without any allocation.  The pages have no
 * counterpart: this entry point exists for callers that cannot call cudaMalloc --
 * code that runs while a CUDA graph is being captured, runtimes whose device memory
 * belongs entirely to their own pool allocator, embedded users that forbid allocation
 * after start-up -- and so cannot build a handle with sfnn_create.
 *   x  [d], pa = A [d x r], pb = B [r x n], pc = c [n]: DEVICE, PyTorch layouts, wdtype
 *   idx [n] int32 out: the selected neurons in ascending order (first *count entries)
 *   count [1] int32 out
 * The set is S(x) = { i : (relu(x.A).B + c)_i > 0 }, as sfnn_predict computes it.
 * Scratch (the hidden layer and the decision mask) lives in one static device array
 * of SFNN_NOALLOC_SCRATCH_BYTES that every GPU loading the library holds until exit;
 * the call needs 4*r rounded up to 256, plus 4*ceil(n/32) bytes of it, and returns
 * SFNN_ERR_UNSUPPORTED, launching nothing, when r and n need more.  It calls no
 * allocation routine.  The first call on a device looks up that device's address of
 * the array (cudaGetSymbolAddress); make it before any stream capture.  The address
 * is kept for the life of the process: a cudaDeviceReset of that device frees the
 * array with its context, and the entry point must not be called on it again.  Every call
 * shares the array: calls that overlap on the GPU (other streams, other host threads)
 * race and must be serialised by the caller.  Asynchronous on `stream`.
 */
#define SFNN_NOALLOC_SCRATCH_BYTES (64 * 1024)
SFNN_API sfnn_status sfnn_predict_noalloc(const void *x, const void *pa, const void *pb, const void *pc, int32_t d,
                                          int32_t r, int32_t n, int32_t wdtype, int32_t *idx, int32_t *count,
                                          sfnn_stream_t stream);

/* Fill *info (host struct). */
SFNN_API sfnn_status sfnn_query(sfnn_handle h, sfnn_info *info);

/* Return and clear the latched device-side error of h (synchronises h's device). */
SFNN_API sfnn_status sfnn_get_error(sfnn_handle h);

/* Static description of a status code; never NULL. */
SFNN_API const char *sfnn_status_str(sfnn_status s);

/*
 * Host only: the storage order sfnn_create uses.  perm[k] = the neuron stored
 * at position k: hotness descending, ties by ascending index, NaN last.
 *   hotness [n] HOST in;  perm [n] HOST out.
 */
SFNN_API sfnn_status sfnn_hotness_order(const float *hotness, int32_t n, int32_t *perm);

#ifdef __cplusplus
}
#endif

#endif /* SFNN_H */
