/*
 * moe.h -- C ABI of libmoe.so, a B200 (sm_100a) fused Mixture-of-Experts layer forward.
 *
 * The operation (per token t, hidden size H, E routed experts, top-k K):
 *   1. router logits    l[t,e] = x[t,:] . Wr[e,:]            (BF16 in, FP32 accumulate)
 *   2. router top-k     "Laguna exact M=8 BF16-input router top-k preregistration",
 *                       section "Question and arithmetic contract": FP32 sigmoid (or
 *                       softmax) scores, an FP32 correction bias used only for selection,
 *                       lower-expert-ID tie break, top K, renormalised unbiased weights.
 *   3. permutation      token slots grouped by expert (FlashInfer PR #4646, walkthrough:
 *                       "routing permutation").
 *   4. FC1 + activation h = SwiGLU(W13[e] x) = silu(gate) * up, or ReLU^2(W1[e] x)
 *                       (FlashInfer PR #4646, description: SwiGLU gated / ReLU2 ungated).
 *   5. FC2 + combine    routed[t] = sum_k w[t,k] * W2[e_k] h[t,k], FP32 accumulation.
 *   6. shared expert    out = bf16( bf16(routed) + bf16(shared FFN(x)) ), the order of
 *                       "MTP1 isolated gather/shared-add closure" (b70-optimization-lab):
 *                       routed FP32 accumulation -> BF16 -> shared BF16 add -> BF16.
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers on the current CUDA device, row-major and
 *     contiguous, 16-byte aligned.  BF16 tensors are raw bfloat16 bit patterns.
 *   - The caller owns every buffer.  The library never allocates, frees or synchronises
 *     (moe_get_error is the one call that synchronises its stream).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream).
 *   - Arguments are validated on the host before anything is enqueued; on error nothing
 *     is launched and the status says why.  T == 0 (moe_fused_forward) and M == 0
 *     (moe_router_topk) return MOE_OK and launch nothing.
 *   - There is no hidden global state: concurrent calls are safe when they use distinct
 *     outputs and workspaces.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size or enum value */
    MOE_ERR_UNSUPPORTED = 2,  /* valid but outside what this build supports (limits below) */
    MOE_ERR_WORKSPACE = 3,    /* workspace missing, misaligned (256 B) or too small */
    MOE_ERR_CUDA = 4,         /* a CUDA runtime call failed (launch, attribute, driver entry) */
    MOE_ERR_DEVICE = 5        /* the device error word is set (see moe_get_error) */
} moe_status_t;

typedef enum { MOE_SCORE_SOFTMAX = 0, MOE_SCORE_SIGMOID = 1 } moe_score_t;
typedef enum { MOE_ACT_SWIGLU = 0, MOE_ACT_RELU2 = 1 } moe_act_t;
typedef enum { MOE_DT_BF16 = 0, MOE_DT_FP32 = 1 } moe_dtype_t;
/* Execution path of moe_fused_forward.  AUTO picks by token count (see
 * moe_select_path).  SMALL streams only the routed experts' weights with CUDA-core dot
 * products spread over all SMs; LARGE runs the grouped tcgen05 tensor-core GEMMs. */
typedef enum { MOE_PATH_AUTO = 0, MOE_PATH_SMALL = 1, MOE_PATH_LARGE = 2 } moe_path_t;

/* Device error codes written to the workspace error word. */
#define MOE_DEVERR_BAD_EXPERT_ID 0x1   /* an expert id outside [0, E) reached the permute */
#define MOE_DEVERR_WAIT_TIMEOUT 0x2    /* a bounded device-side wait gave up */
#define MOE_DEVERR_BAD_INDEX 0x4       /* a computed row/slot index fell outside its buffer; the access was skipped */
#define MOE_DEVERR_ROUTER_BOUND 0x8    /* a tensor-core router logit lay outside its error bound: the
                                          hardware accumulation model behind exact routing did not hold, so
                                          this call's expert ids are not guaranteed to be the exact ones */

/* Limits of this build. */
#define MOE_MAX_EXPERTS 1024
#define MOE_MAX_TOPK 32
#define MOE_MAX_TOKENS 65536

/* ------------------------------------------------------------------------------------
 * moe_router_topk -- router scores + top-k + weights for M rows of logits.
 * Passage: "Laguna exact M=8 BF16-input router top-k preregistration", "Question and
 * arithmetic contract" (BF16 logits -> exact widening -> FP32 sigmoid -> + FP32 bias for
 * selection only -> lower-expert-ID tie break -> top k -> renormalise the unbiased FP32
 * sigmoid weights) and "Four-card component gate" (source index slot * M + row).
 *   logits     [M, E] BF16 (logits_dtype = MOE_DT_BF16) or FP32 (MOE_DT_FP32).
 *   score      MOE_SCORE_SIGMOID: s = sigmoid(l) in FP32 (correctly rounded), key = s + b
 *              (FP32 add).  MOE_SCORE_SOFTMAX: key = l (+ b if bias), weights from the
 *              softmax of the logits.
 *   bias       [E] FP32 or NULL (= zero).  Used for selection only.
 *   renorm     1: weights renormalised over the K selected experts (sigmoid: s_k / sum s;
 *              softmax: exp(l_k - lmax) / sum over the selected); 0: sigmoid -> s_k,
 *              softmax -> full softmax probability over all E.
 *   topk_w     [M, K] FP32 out, slot k = k-th largest key (ties -> lower expert id).
 *   topk_ids   [M, K] int32 out.
 *   src_idx    [M, K] int32 out, src_idx[m,k] = k * M + m.  May be NULL.
 * Limits: 1 <= E <= MOE_MAX_EXPERTS, 1 <= K <= min(E, MOE_MAX_TOPK), 0 <= M.
 * NaN logits are selected last (treated as -inf); their weights are undefined.
 * ---------------------------------------------------------------------------------- */
moe_status_t moe_router_topk(const void* logits, int logits_dtype, int M, int E, int top_k,
                             int score, const float* bias, int renorm, float* topk_w,
                             int32_t* topk_ids, int32_t* src_idx, void* stream);

/* ------------------------------------------------------------------------------------
 * moe_permute -- group the M*K token slots by expert.
 * Passage: FlashInfer PR #4646, walkthrough (routing permutation) and review notes on
 * the permute scan (padded-count reduction, exclusive scan, per-expert offsets).  This
 * build is unpadded and deterministic.
 *   topk_ids        [M, K] int32 in; ids must lie in [0, E).
 *   expert_offsets  [E + 1] int32 out: exclusive prefix sum of the per-expert counts,
 *                   expert_offsets[E] = M * K.
 *   perm            [M * K] int32 out: source indices src = k * M + m, grouped by expert
 *                   in ascending expert order and by ascending token m within an expert.
 *   inv             [M * K] int32 out: inv[src] = position of src in perm.  May be NULL.
 *   ws, ws_bytes    device workspace of at least moe_permute_workspace_size(M, K, E) bytes,
 *                   256-byte aligned.  Holds the device error word.
 * M == 0 still writes expert_offsets (all zero).
 * An id outside [0, E) sets MOE_DEVERR_BAD_EXPERT_ID in the error word (read it with
 * moe_get_error); that slot is left out of perm and the outputs are then incomplete.
 * Limits: M * K <= MOE_MAX_TOKENS * 8, E <= MOE_MAX_EXPERTS, K <= MOE_MAX_TOPK.
 * ---------------------------------------------------------------------------------- */
size_t moe_permute_workspace_size(int M, int K, int E);
moe_status_t moe_permute(const int32_t* topk_ids, int M, int K, int E, int32_t* expert_offsets,
                         int32_t* perm, int32_t* inv, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------------------
 * moe_fused_forward -- the whole layer (steps 1-6 above) for T tokens.
 * Layer description: */
typedef struct {
    int T;            /* tokens, 0 <= T <= MOE_MAX_TOKENS */
    int H;            /* hidden size, multiple of 8 */
    int I;            /* routed-expert intermediate size, multiple of 8 */
    int E;            /* routed experts, 1..MOE_MAX_EXPERTS */
    int top_k;        /* 1..min(E, MOE_MAX_TOPK) */
    int act;          /* moe_act_t */
    int score;        /* moe_score_t */
    int renorm;       /* 0 or 1, as in moe_router_topk */
    int I_shared;     /* shared-expert intermediate size (multiple of 8), 0 = none */
    int path;         /* moe_path_t */
    const void* router_w;        /* [E, H] BF16; may be NULL when router_logits is given */
    const float* router_logits;  /* [T, E] FP32 logits to route on instead of x . Wr^T, or NULL */
    const float* bias;           /* [E] FP32 selection bias or NULL */
    const void* w13;             /* SwiGLU: [E, 2I, H] BF16, rows [0,I) gate, [I,2I) up;
                                    ReLU^2: [E, I, H] BF16 */
    const void* w2;              /* [E, H, I] BF16 */
    const void* ws13;            /* shared expert, [2I_s, H] or [I_s, H] BF16, or NULL */
    const void* ws2;             /* shared expert, [H, I_s] BF16, or NULL */
    /* Optional parts of the layer; a zero-initialised field leaves the plain layer.
     *  routed_scale   the routed FP32 sum is multiplied by it before its BF16 rounding
     *                 (a routed scaling factor applied to the routed output after the
     *                 router, as "Laguna exact M=8 BF16-input router top-k
     *                 preregistration", "Question and arithmetic contract", describes);
     *                 0 means 1.  Must be finite.
     *  shared_gate_w  [H] BF16 gate row of the internal shared expert (needs I_shared > 0)
     *                 or NULL: the shared output of token t is multiplied by
     *                 g_t = sigmoid(x[t] . w) (an FP32 logit of the exact products, the
     *                 router's correctly rounded FP32 sigmoid) before its BF16 rounding --
     *                 the (1, H) shared-expert gate of vLLM PR #64636's decode table.
     *  shared_out     [T, H] BF16 shared-expert output computed by the caller, or NULL;
     *                 only with I_shared == 0.  It is added in place of an internal shared
     *                 expert, in the same order (routed BF16, then the BF16 add).  `out`
     *                 may be this very buffer (the in-place, shared-output-alias form of
     *                 "MTP1 isolated gather/shared-add closure"); it must not overlap it
     *                 otherwise. */
    float routed_scale;
    const void* shared_gate_w;
    const void* shared_out;
    /* Optional phase trace (NULL = none): a device buffer of moe_trace_size() bytes that the
     * tensor-core kernels of the many-token path fill, one block per kernel (MOE_TRACE_ROUTER,
     * _FC1, _FC2), one row of MOE_TRACE_FIELDS 64-bit values per CTA: %globaltimer (ns) at
     * kernel entry, when its inputs are ready (after the wait on the previous kernel and the
     * tile tables), when its producer issued its last load, when its first epilogue warp
     * finished, and at exit; and the number of work units (tiles, or stream-K segments) the
     * CTA took.  Rows of CTAs a kernel did not launch, and blocks of kernels the call did
     * not run, are left as they were.  16-byte aligned. */
    unsigned long long* trace;
    /* Tile schedule of the many-token path's grouped GEMMs (moe_sched_t): STATIC deals the
     * tiles round-robin over the persistent CTAs; DYNAMIC lets each CTA take the next tile
     * of the same list from a device counter whenever its load pipeline is ready for one;
     * AUTO (0) chooses per call.  Results are identical up to the FP32 order of the
     * routed combine (already unspecified).  GEMMs that run stream-K (few-token calls)
     * keep their own schedule. */
    int schedule;
    /* Token rows per tile of the many-token path's grouped GEMMs, 0 = chosen per call from
     * the average rows per expert (moe_token_tiles reports the choice).  FC1: 32, 64, 128,
     * or 256 (ReLU^2 only); FC2: 32, 128, 192 or 256; anything else is MOE_ERR_INVALID_ARG.
     * For tuning: results do not depend on it beyond the FP32 order of the routed combine. */
    int fc1_tile_rows, fc2_tile_rows;
} moe_layer_desc;

typedef enum { MOE_SCHED_AUTO = 0, MOE_SCHED_STATIC = 1, MOE_SCHED_DYNAMIC = 2 } moe_sched_t;

enum { MOE_TRACE_ENTRY = 0, MOE_TRACE_READY = 1, MOE_TRACE_LOADS_DONE = 2, MOE_TRACE_STORES_DONE = 3,
       MOE_TRACE_EXIT = 4, MOE_TRACE_UNITS = 5, MOE_TRACE_FIELDS = 8 };
enum { MOE_TRACE_ROUTER = 0, MOE_TRACE_FC1 = 1, MOE_TRACE_FC2 = 2, MOE_TRACE_KERNELS = 3 };
#define MOE_TRACE_MAX_CTAS 1024
/* Bytes of the phase-trace buffer: MOE_TRACE_KERNELS blocks of MOE_TRACE_MAX_CTAS rows. */
size_t moe_trace_size(void);

/* Bytes of workspace moe_fused_forward needs for this description (either path). */
size_t moe_workspace_size(const moe_layer_desc* d);

/* Path MOE_PATH_AUTO resolves to for this description (MOE_PATH_SMALL or _LARGE). */
int moe_select_path(const moe_layer_desc* d);

/*   x            [T, H] BF16 in.
 *   out          [T, H] BF16 out; must not overlap x or any weight, and may overlap
 *                d->shared_out only by being exactly that buffer.
 *   topk_w_out   [T, K] FP32 out or NULL (routing weights, as moe_router_topk).
 *   topk_ids_out [T, K] int32 out or NULL.
 *   logits_out   [T, E] FP32 out or NULL (the router logits used; a copy of
 *                router_logits when those are given).
 *   ws, ws_bytes workspace of at least moe_workspace_size(d) bytes, 256-byte aligned;
 *                its first 256 bytes hold the device error word.
 * The shared expert uses the routed activation; its sigmoid gate is optional (shared_gate_w).
 * Routing is exact: expert ids and weights are those of the exact logits (the FP32
 * rounding of the exact sum of the BF16 products, up to an FP64 summation error far
 * below an FP32 unit).  Up to 64 tokens the logits are computed that way directly.  With
 * more tokens a tensor-core GEMM screens them; every expert whose key lies within twice
 * a per-token error bound of the K-th key is re-evaluated exactly, so no expert outside
 * that window can belong to the top K.  The bound models each 16-product step of the
 * tensor core's FP32 accumulation as aligning its addends to the largest and keeping at
 * least 24 bits of it; a re-evaluated logit found outside the bound sets
 * MOE_DEVERR_ROUTER_BOUND (read it with moe_get_error). */
moe_status_t moe_fused_forward(const moe_layer_desc* d, const void* x, void* out,
                               float* topk_w_out, int32_t* topk_ids_out, float* logits_out,
                               void* ws, size_t ws_bytes, void* stream);

/* Number of kernels moe_fused_forward enqueues for this description (for accounting). */
int moe_fused_forward_launches(const moe_layer_desc* d);

/* The kernels moe_fused_forward enqueues for this description, in launch order: writes up
 * to max_kernels MOE_K_* values to `kernels` (may be NULL) and returns their number (0
 * for an invalid description or T == 0).  The path and the router used decide the list. */
enum { MOE_K_PREP = 0,        /* zero the call's counters; bound the router rows' norms */
       MOE_K_ROUTER = 1,      /* router logits */
       MOE_K_ROUTE_TABLE = 2, /* few-token path: routing and the distinct-expert table */
       MOE_K_TOPK = 3,        /* top-k (screening, exact re-evaluation, selection), or its screen */
       MOE_K_TOPK_REFINE = 4, /* split top-k: exact re-evaluation of the candidates */
       MOE_K_TOPK_SELECT = 5, /* split top-k: selection on exact keys */
       MOE_K_PERMUTE = 6, MOE_K_FC1 = 7, MOE_K_FC2 = 8, MOE_K_FINALIZE = 9 };
int moe_fused_forward_plan(const moe_layer_desc* d, int* kernels, int max_kernels);

/* Token rows per tile of the many-token path's grouped GEMMs for this description (the
 * MMA N of one tile: FC1 and FC2 each pick one width per call from T * top_k / E).
 * Returns MOE_OK, or the description's validation error. */
moe_status_t moe_token_tiles(const moe_layer_desc* d, int* fc1_rows, int* fc2_rows);

/* Where moe_fused_forward keeps an intermediate in the workspace, for inspection after a
 * call (tests, debugging).  Valid after a many-token-path (MOE_PATH_LARGE) call with this
 * description, until the workspace is reused:
 *   MOE_WS_TOPK_IDS  [T, K] int32 expert ids      MOE_WS_TOPK_W  [T, K] FP32 weights
 *   MOE_WS_OFFSETS   [E + 1] int32 expert offsets of the internal permutation
 *   MOE_WS_PERM      [T * K] int32 source slots k * T + t grouped by expert (the order
 *                    within an expert is unspecified; the set of each expert is exact)
 * Writes the region's byte offset from the workspace start and its size. */
enum { MOE_WS_TOPK_IDS = 0, MOE_WS_TOPK_W = 1, MOE_WS_OFFSETS = 2, MOE_WS_PERM = 3 };
moe_status_t moe_workspace_region(const moe_layer_desc* d, int region, size_t* offset, size_t* bytes);

/* moe_fused_forward with per-kernel timing: `events` holds n_events >= launches + 1
 * cudaEvent_t handles created by the caller; event i is recorded on `stream` before the
 * i-th kernel and event `launches` after the last.  Recording events between the kernels
 * disables their programmatic overlap, so this variant is for attribution, not for the
 * headline timing.  Same arguments and errors as moe_fused_forward, plus
 * MOE_ERR_INVALID_ARG when n_events is too small. */
moe_status_t moe_fused_forward_timed(const moe_layer_desc* d, const void* x, void* out, float* topk_w_out,
                                     int32_t* topk_ids_out, float* logits_out, void* ws, size_t ws_bytes,
                                     void* stream, void* const* events, int n_events);

/* ------------------------------------------------------------------------------------
 * moe_fused_forward_noalloc -- moe_fused_forward for callers that cannot allocate.
 * The pages have no counterpart: this is a deployment variant of this library.
 * Some callers cannot allocate device memory at the point where they run the layer:
 * code that runs while a CUDA graph is being captured (allocation calls are not
 * capturable), runtimes that hand out a fixed memory pool and forbid further
 * cudaMalloc, or plugins whose host framework owns every allocation.  This entry point
 * takes the same description and buffers as moe_fused_forward minus the workspace: its
 * scratch is a static device array of MOE_NOALLOC_SCRATCH_BYTES inside libmoe.so
 * (every GPU that loads the library holds it until the process exits).  It allocates
 * nothing and frees nothing.
 *   - Returns MOE_ERR_WORKSPACE, before launching anything, when the description needs
 *     more scratch than that (moe_workspace_size(d) > MOE_NOALLOC_SCRATCH_BYTES); the
 *     other errors are those of moe_fused_forward.
 *   - The first call on each device (with that device current) looks up the array's
 *     device address and clears its error word; make that first call before any
 *     stream capture begins.  The lookup is repeated when the device's CUDA context
 *     changes (after cudaDeviceReset).
 *   - All calls on a device share the array: calls whose GPU work overlaps (different
 *     streams, concurrent graph launches) race and give wrong results.
 *   - Device error flags (MOE_DEVERR_*) accumulate in the array's error word over calls
 *     until moe_noalloc_get_error reads and clears them.
 * ---------------------------------------------------------------------------------- */
#define MOE_NOALLOC_SCRATCH_BYTES (16u << 20)
moe_status_t moe_fused_forward_noalloc(const moe_layer_desc* d, const void* x, void* out,
                                       float* topk_w_out, int32_t* topk_ids_out, float* logits_out,
                                       void* stream);

/* moe_noalloc_get_error -- moe_get_error for the static scratch of the current device:
 * reads and clears the error word that moe_fused_forward_noalloc calls on this device
 * write.  Synchronises `stream`; allocates nothing (on a device with no call yet, it sets
 * the array up as the first call would).
 *   code  out: OR of MOE_DEVERR_* flags set since the last read (0 = none).
 * Returns MOE_ERR_DEVICE when code != 0, MOE_OK otherwise, MOE_ERR_CUDA if a CUDA call
 * fails, MOE_ERR_INVALID_ARG when code is NULL. */
moe_status_t moe_noalloc_get_error(int* code, void* stream);

/* ------------------------------------------------------------------------------------
 * moe_get_error -- read and clear the device error word at the start of `ws`
 * (a moe_fused_forward or moe_permute workspace).  Synchronises `stream`.
 *   code  out: OR of MOE_DEVERR_* flags set since the last read (0 = none).
 * Returns MOE_ERR_DEVICE when code != 0, MOE_OK otherwise, MOE_ERR_CUDA if the copy fails.
 * ---------------------------------------------------------------------------------- */
moe_status_t moe_get_error(void* ws, int* code, void* stream);

/* Human-readable name of a status code (static storage). */
const char* moe_status_string(moe_status_t s);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
