// api.cu -- the C ABI of libmoe.so: host-side validation, workspace layout, path
// selection, tensor-map encoding and the launch sequence of each path.  Nothing here
// allocates or synchronises device memory (except moe_get_error).
#include <cstring>

#include "kernels.cuh"

using namespace moe;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

// SMs of the current device (148 on B200; also the value used without a device).
int num_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}

// Workspace carve-up of moe_fused_forward, 256-byte aligned regions after the header.
struct WsLayout {
    size_t logits, route, topk_w, topk_ids, offsets, tiles1, tiles2, counts, perm, cand, h, hs, acc, done, wpart, xn2,
        roweps, skp, gate, total;
};
// Candidate-list capacity per token of the three-kernel top-k (rows with more fall back).
constexpr size_t kCandPerRow = 32;
// Counters zeroed at the start of each many-token call (by its first kernel): per-expert
// counts, per-expert cursors, the candidate count; and, in a region of their own, FC1's
// stream-K per-tile counters.
inline size_t counter_ints(size_t E) { return 2 * (E + 2) + 4; }
inline size_t cand_count_int(size_t E) { return 2 * (E + 2); }
// Next-tile counters of the dynamic schedule (FC1: which = 0, FC2: 1).
inline size_t dyn_count_int(size_t E, int which) { return 2 * (E + 2) + 1 + which; }
// Token rows per grouped-GEMM tile of a call: the caller's choice, else by rows per expert.
int fc1_tile_rows(const moe_layer_desc* d) {
    if (d->fc1_tile_rows) return d->fc1_tile_rows;
    return gemm_token_tile(d->act == MOE_ACT_SWIGLU ? GM_FC1_SWIGLU : GM_FC1_RELU2, d->T, d->top_k, d->E);
}
int fc2_tile_rows(const moe_layer_desc* d) {
    return d->fc2_tile_rows ? d->fc2_tile_rows : gemm_token_tile(GM_FC2, d->T, d->top_k, d->E);
}
// Per-CTA router weight-norm bounds of the prep kernel (one per SM at most).
constexpr size_t kMaxPrepGrid = 1024;
WsLayout layout(const moe_layer_desc* d) {
    const size_t T = (size_t)d->T, E = (size_t)d->E, K = (size_t)d->top_k, H = (size_t)d->H, I = (size_t)d->I,
                 Is = (size_t)d->I_shared;
    WsLayout L;
    size_t o = kHeaderBytes;
    auto take = [&](size_t bytes) {
        const size_t r = o;
        o = align_up(o + bytes, 256);
        return r;
    };
    L.logits = take(T * E * 4);
    L.route = take(sizeof(RouteTable));
    L.topk_w = take(T * K * 4);
    L.topk_ids = take(T * K * 4);
    L.offsets = take((E + 2) * 4);
    L.tiles1 = take((E + 2) * 4);
    L.tiles2 = take((E + 2) * 4);
    L.counts = take(counter_ints(E) * 4);
    L.perm = take(T * K * 4);
    L.cand = take(T * (2 + 3 * kCandPerRow) * 4);  // row_base, row_n, cand_row, cand_e, cand_val
    L.h = take(T * K * I * 2);
    L.hs = take(T * Is * 2);
    L.acc = take(T * H * 4 * (Is ? 2 : 1));  // routed sum, then the shared expert's (FP32)
    // Small regions after the large ones, so that the large buffers keep their offsets.
    L.done = take((size_t)kStreamKMaxTiles * 4);
    L.wpart = take(kMaxPrepGrid * 4);
    L.xn2 = take(T * 4);
    L.roweps = take(T * 4);
    L.skp = take(fc1_streamk_bytes(fc1_tile_rows(d), d->act == MOE_ACT_SWIGLU, num_sms()));
    L.gate = take(d->shared_gate_w ? T * 4 : 0);
    L.total = o;
    return L;
}

moe_status_t validate_desc(const moe_layer_desc* d) {
    if (!d) return MOE_ERR_INVALID_ARG;
    if (d->T < 0 || d->H < 8 || d->I < 8 || d->E < 1 || d->top_k < 1) return MOE_ERR_INVALID_ARG;
    if (d->H % 8 || d->I % 8 || d->I_shared < 0 || d->I_shared % 8) return MOE_ERR_INVALID_ARG;
    if (d->act != MOE_ACT_SWIGLU && d->act != MOE_ACT_RELU2) return MOE_ERR_INVALID_ARG;
    if (d->score != MOE_SCORE_SOFTMAX && d->score != MOE_SCORE_SIGMOID) return MOE_ERR_INVALID_ARG;
    if (d->renorm != 0 && d->renorm != 1) return MOE_ERR_INVALID_ARG;
    if (d->path < MOE_PATH_AUTO || d->path > MOE_PATH_LARGE) return MOE_ERR_INVALID_ARG;
    if (d->top_k > d->E) return MOE_ERR_INVALID_ARG;
    if (d->E > MOE_MAX_EXPERTS || d->top_k > MOE_MAX_TOPK || d->T > MOE_MAX_TOKENS) return MOE_ERR_UNSUPPORTED;
    if (d->I_shared > 0 && d->E + 1 > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
    if (!d->router_w && !d->router_logits) return MOE_ERR_INVALID_ARG;
    if (!d->w13 || !d->w2) return MOE_ERR_INVALID_ARG;
    if (d->I_shared > 0 && (!d->ws13 || !d->ws2)) return MOE_ERR_INVALID_ARG;
    if (!(d->routed_scale == d->routed_scale) || d->routed_scale > 3.4e38f || d->routed_scale < -3.4e38f)
        return MOE_ERR_INVALID_ARG;  // NaN or infinite
    if (d->shared_gate_w && d->I_shared == 0) return MOE_ERR_INVALID_ARG;
    if (d->shared_out && d->I_shared > 0) return MOE_ERR_INVALID_ARG;
    if (d->schedule < MOE_SCHED_AUTO || d->schedule > MOE_SCHED_DYNAMIC) return MOE_ERR_INVALID_ARG;
    const int t1 = d->fc1_tile_rows, t2 = d->fc2_tile_rows;
    if (t1 && t1 != 32 && t1 != 64 && t1 != 128 && !(t1 == 256 && d->act == MOE_ACT_RELU2))
        return MOE_ERR_INVALID_ARG;
    if (t2 && t2 != 32 && t2 != 128 && t2 != 192 && t2 != 256) return MOE_ERR_INVALID_ARG;
    const void* ptrs[] = {d->router_w, d->router_logits, d->bias, d->w13, d->w2, d->ws13, d->ws2,
                          d->shared_gate_w, d->shared_out, d->trace};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

// Byte ranges [a, a + na) and [b, b + nb) overlap.
bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

// Token-count rule of MOE_PATH_AUTO.  The streaming path reads each routed expert once
// and wins while the experts see few tokens; the tensor-core path wins once its MMA
// work per weight byte pays for the tile machinery.
// Path selector.  The streaming path saves the many-token path's extra kernels (top-k +
// permute + finalize against one route-table kernel), but streams weights on the CUDA
// cores more slowly than TMA + tcgen05 does, so it wins only while the weight bytes of
// the call are small.  The threshold sits in the measured crossover on B200: the
// streaming path was ahead at 100.7 MB of touched expert weights (Qwen3.6-shaped T = 2)
// and behind at 108 MB (large-E-shaped T = 1, with its shared expert) and above.
static constexpr double kSmallPathMaxBytes = 104e6;
// The streaming path routes on exact logits: given ones, or the few-token router's.
bool small_path_ok(const moe_layer_desc* d) {
    return small_path_supported(d->T, d->H, d->I, d->I_shared) && (d->router_logits || router_small_supported(d->H));
}
int auto_path(const moe_layer_desc* d) {
    if (!small_path_ok(d)) return MOE_PATH_LARGE;
    const double m = d->act == MOE_ACT_SWIGLU ? 3.0 : 2.0;
    const double experts = (double)std::min(d->T * d->top_k, d->E);
    const double bytes = experts * m * d->H * d->I * 2.0 + m * d->H * (double)d->I_shared * 2.0;
    return bytes <= kSmallPathMaxBytes ? MOE_PATH_SMALL : MOE_PATH_LARGE;
}
int resolve_path(const moe_layer_desc* d) {
    if (d->path == MOE_PATH_AUTO) return auto_path(d);
    return d->path;
}
// Tile schedule of the many-token path's grouped GEMMs (GEMMs that run stream-K keep
// theirs).  AUTO takes the dynamic schedule from 256 average rows per expert on: there the
// round-robin left the CTAs' finishing times 100-150 us apart (Qwen3.6-shaped T = 8192:
// 775 -> 767 us; Nemotron-shaped T = 8192: 1520 -> 1481 us), while below it the dynamic
// kernel's FC2 is slower than its tail saving (Qwen3.6-shaped T = 4096: 440 -> 468 us).
int resolve_schedule(const moe_layer_desc* d) {
    if (d->schedule != MOE_SCHED_AUTO) return d->schedule;
    return (long long)d->T * d->top_k >= 256LL * d->E ? MOE_SCHED_DYNAMIC : MOE_SCHED_STATIC;
}


// ---------------------------------------------------------------- tensor maps
bool map2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows) {
    EncodeTiledFn enc = get_encode_tiled();
    if (!enc) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
bool map3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t depth, uint32_t box_rows) {
    EncodeTiledFn enc = get_encode_tiled();
    if (!enc) return false;
    cuuint64_t dims[3] = {inner, rows, depth};
    cuuint64_t strides[2] = {inner * 2, inner * rows * 2};
    cuuint32_t box[3] = {64, box_rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

#define MOE_CK(x)                                 \
    do {                                          \
        if ((x) != cudaSuccess) return MOE_ERR_CUDA; \
    } while (0)

// Router logits x . Wr^T on the tensor cores for many tokens (A = Wr, B = x rows).
moe_status_t run_router_dense(const moe_layer_desc* d, const bf16* x, float* logits, float* copy, int sms,
                              cudaStream_t s, int* err, bool pdl) {
    GemmArgs g;
    std::memset(&g, 0, sizeof(g));
    g.T = d->T;
    g.kdim = d->H;
    g.nfeat_r = cdiv(d->E, 128);
    g.feat_r = d->E;
    g.E = 1;
    g.dense = 1;
    g.logits = logits;
    g.logits_copy = copy;
    g.trace = d->trace ? d->trace + (size_t)MOE_TRACE_ROUTER * MOE_TRACE_MAX_CTAS * MOE_TRACE_FIELDS : nullptr;
    g.err = err;
    GemmMaps m;
    std::memset(&m, 0, sizeof(m));
    if (!map2d(&m.a_r, d->router_w, d->H, d->E, 128) || !map2d(&m.b_r, x, d->H, d->T, 16)) return MOE_ERR_CUDA;
    m.a_s = m.a_r;
    m.b_s = m.b_r;
    const int tiles = g.nfeat_r * cdiv(d->T, kDenseTokenTile);
    MOE_CK(launch_gemm(GM_DENSE, 0, g, m, std::min(sms, tiles), s, pdl));
    return MOE_OK;
}

}  // namespace

namespace moe {
EncodeTiledFn get_encode_tiled() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}
}  // namespace moe

extern "C" {

const char* moe_status_string(moe_status_t s) {
    switch (s) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
        case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
        case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
        case MOE_ERR_DEVICE: return "MOE_ERR_DEVICE";
    }
    return "MOE_ERR_UNKNOWN";
}

moe_status_t moe_router_topk(const void* logits, int logits_dtype, int M, int E, int top_k, int score,
                             const float* bias, int renorm, float* topk_w, int32_t* topk_ids, int32_t* src_idx,
                             void* stream) {
    if (M < 0 || E < 1 || top_k < 1 || top_k > E) return MOE_ERR_INVALID_ARG;
    if (logits_dtype != MOE_DT_BF16 && logits_dtype != MOE_DT_FP32) return MOE_ERR_INVALID_ARG;
    if (score != MOE_SCORE_SOFTMAX && score != MOE_SCORE_SIGMOID) return MOE_ERR_INVALID_ARG;
    if (renorm != 0 && renorm != 1) return MOE_ERR_INVALID_ARG;
    if (E > MOE_MAX_EXPERTS || top_k > MOE_MAX_TOPK) return MOE_ERR_UNSUPPORTED;
    if (M == 0) return MOE_OK;
    if (!logits || !topk_w || !topk_ids) return MOE_ERR_INVALID_ARG;
    const void* ptrs[] = {logits, bias, topk_w, topk_ids, src_idx};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return MOE_ERR_INVALID_ARG;
    if (launch_topk(logits, logits_dtype == MOE_DT_BF16, M, E, top_k, score, bias, renorm, topk_w, topk_ids, src_idx,
                    nullptr, nullptr, (cudaStream_t)stream, false) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

size_t moe_permute_workspace_size(int M, int K, int E) {
    (void)M;
    (void)K;
    (void)E;
    return kHeaderBytes;
}

moe_status_t moe_permute(const int32_t* topk_ids, int M, int K, int E, int32_t* expert_offsets, int32_t* perm,
                         int32_t* inv, void* ws, size_t ws_bytes, void* stream) {
    if (M < 0 || K < 1 || E < 1) return MOE_ERR_INVALID_ARG;
    if (E > MOE_MAX_EXPERTS || K > MOE_MAX_TOPK || (long long)M * K > (long long)MOE_MAX_TOKENS * 8)
        return MOE_ERR_UNSUPPORTED;
    if (!ws || !aligned256(ws) || ws_bytes < moe_permute_workspace_size(M, K, E)) return MOE_ERR_WORKSPACE;
    if (!expert_offsets || (M > 0 && (!topk_ids || !perm))) return MOE_ERR_INVALID_ARG;
    const void* ptrs[] = {topk_ids, expert_offsets, perm, inv};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return MOE_ERR_INVALID_ARG;
    PermuteArgs a;
    std::memset(&a, 0, sizeof(a));
    a.ids = topk_ids;
    a.M = M;
    a.K = K;
    a.E = E;
    a.offsets = expert_offsets;
    a.perm = perm;
    a.inv = inv;
    a.err = &static_cast<WsHeader*>(ws)->err;
    if (launch_permute(a, (cudaStream_t)stream, false) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
}

size_t moe_workspace_size(const moe_layer_desc* d) {
    if (validate_desc(d) != MOE_OK) return 0;
    return layout(d).total;
}

int moe_select_path(const moe_layer_desc* d) {
    if (validate_desc(d) != MOE_OK) return -1;
    return resolve_path(d);
}

size_t moe_trace_size(void) {
    return (size_t)MOE_TRACE_KERNELS * MOE_TRACE_MAX_CTAS * MOE_TRACE_FIELDS * sizeof(unsigned long long);
}

moe_status_t moe_token_tiles(const moe_layer_desc* d, int* fc1_rows, int* fc2_rows) {
    const moe_status_t st = validate_desc(d);
    if (st != MOE_OK) return st;
    if (!fc1_rows || !fc2_rows) return MOE_ERR_INVALID_ARG;
    *fc1_rows = fc1_tile_rows(d);
    *fc2_rows = fc2_tile_rows(d);
    return MOE_OK;
}

moe_status_t moe_workspace_region(const moe_layer_desc* d, int region, size_t* offset, size_t* bytes) {
    const moe_status_t st = validate_desc(d);
    if (st != MOE_OK) return st;
    if (!offset || !bytes) return MOE_ERR_INVALID_ARG;
    const WsLayout L = layout(d);
    const size_t TK = (size_t)d->T * d->top_k;
    switch (region) {
        case MOE_WS_TOPK_IDS: *offset = L.topk_ids; *bytes = TK * 4; return MOE_OK;
        case MOE_WS_TOPK_W: *offset = L.topk_w; *bytes = TK * 4; return MOE_OK;
        case MOE_WS_OFFSETS: *offset = L.offsets; *bytes = ((size_t)d->E + 1) * 4; return MOE_OK;
        case MOE_WS_PERM: *offset = L.perm; *bytes = TK * 4; return MOE_OK;
    }
    return MOE_ERR_INVALID_ARG;
}

// The tensor-core router runs when the logits are not given and the few-token router does
// not apply.  Its top-k is split in three kernels for more than 256 experts: there the
// one-kernel top-k, whose warps hold 16+ logits each and refine their candidates one after
// another, runs at low occupancy (measured at E = 512, T = 4096: 97 -> 83 us; at E <= 256 the
// extra launches cost more than they save).  Softmax without renorm keeps the one-kernel
// form, whose weights need every logit of the row.
static bool dense_router_for(const moe_layer_desc* d) {
    return !d->router_logits && !(d->T <= 64 && router_small_supported(d->H));
}
static bool split_topk_mode(const moe_layer_desc* d) {
    return d->E > 256 && (d->score == MOE_SCORE_SIGMOID || d->renorm);
}

// The many-token path's prep kernel runs before the tensor-core router and when the
// logits are given; the few-token router zeroes the counters itself.
static bool prep_kernel_for(const moe_layer_desc* d) { return d->router_logits || dense_router_for(d); }

int moe_fused_forward_plan(const moe_layer_desc* d, int* kernels, int max_kernels) {
    if (validate_desc(d) != MOE_OK || d->T == 0) return 0;
    int k[16], n = 0;
    if (resolve_path(d) == MOE_PATH_SMALL) {
        if (!d->router_logits) k[n++] = MOE_K_ROUTER;
        k[n++] = MOE_K_ROUTE_TABLE;
        k[n++] = MOE_K_FC1;
        k[n++] = MOE_K_FC2;
    } else {
        if (prep_kernel_for(d)) k[n++] = MOE_K_PREP;
        if (!d->router_logits) k[n++] = MOE_K_ROUTER;
        k[n++] = MOE_K_TOPK;
        if (dense_router_for(d) && split_topk_mode(d)) {
            k[n++] = MOE_K_TOPK_REFINE;
            k[n++] = MOE_K_TOPK_SELECT;
        }
        k[n++] = MOE_K_PERMUTE;
        k[n++] = MOE_K_FC1;
        k[n++] = MOE_K_FC2;
        k[n++] = MOE_K_FINALIZE;
    }
    for (int i = 0; kernels && i < n && i < max_kernels; ++i) kernels[i] = k[i];
    return n;
}

int moe_fused_forward_launches(const moe_layer_desc* d) { return moe_fused_forward_plan(d, nullptr, 0); }

static moe_status_t fused_forward_impl(const moe_layer_desc* d, const void* x_, void* out_, float* topk_w_out,
                                       int32_t* topk_ids_out, float* logits_out, void* ws, size_t ws_bytes,
                                       void* stream, void* const* events, int n_events) {
    moe_status_t st = validate_desc(d);
    if (st != MOE_OK) return st;
    if (d->T == 0) return MOE_OK;
    if (!x_ || !out_ || !aligned16(x_) || !aligned16(out_)) return MOE_ERR_INVALID_ARG;
    if ((topk_w_out && !aligned16(topk_w_out)) || (topk_ids_out && !aligned16(topk_ids_out)) ||
        (logits_out && !aligned16(logits_out)))
        return MOE_ERR_INVALID_ARG;
    const size_t act_bytes = (size_t)d->T * d->H * 2;
    if (overlaps(out_, act_bytes, x_, act_bytes)) return MOE_ERR_INVALID_ARG;
    if (d->shared_out && out_ != d->shared_out && overlaps(out_, act_bytes, d->shared_out, act_bytes))
        return MOE_ERR_INVALID_ARG;  // in place only as the very same buffer
    const WsLayout L = layout(d);
    if (!ws || !aligned256(ws) || ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    const int path = resolve_path(d);
    if (path == MOE_PATH_SMALL && !small_path_ok(d)) return MOE_ERR_UNSUPPORTED;

    cudaStream_t s = (cudaStream_t)stream;
    if (events && n_events < moe_fused_forward_launches(d) + 1) return MOE_ERR_INVALID_ARG;
    int ev_i = 0;
    // Records the next timing event (between kernels) when the caller asked for them.
    auto mark = [&]() -> bool {
        if (!events) return true;
        return cudaEventRecord((cudaEvent_t)events[ev_i++], s) == cudaSuccess;
    };
    const bool timed = events != nullptr;
    uint8_t* w8 = static_cast<uint8_t*>(ws);
    int* err = &static_cast<WsHeader*>(ws)->err;
    const bf16* x = static_cast<const bf16*>(x_);
    bf16* out = static_cast<bf16*>(out_);
    const int T = d->T, H = d->H, I = d->I, E = d->E, K = d->top_k, Is = d->I_shared;
    const int sms = num_sms();
    if (d->trace && sms > MOE_TRACE_MAX_CTAS) return MOE_ERR_UNSUPPORTED;
    const float rscale = d->routed_scale == 0.0f ? 1.0f : d->routed_scale;
    const bf16* sh_out = static_cast<const bf16*>(d->shared_out);

    // 0. many-token path: the prep kernel zeroes the slot counters and, before the
    // tensor-core router, bounds the router rows' norms.  It is the call's first kernel
    // (no programmatic overlap with the work before the call).
    const bool dense_router = path == MOE_PATH_LARGE && dense_router_for(d);
    float* wpart = reinterpret_cast<float*>(w8 + L.wpart);
    bool pdl = false;
    if (path == MOE_PATH_LARGE && prep_kernel_for(d)) {
        if (!mark()) return MOE_ERR_CUDA;
        MOE_CK(launch_prep(reinterpret_cast<int*>(w8 + L.counts), (int)counter_ints(E),
                           reinterpret_cast<int*>(w8 + L.done), kStreamKMaxTiles,
                           dense_router ? static_cast<const bf16*>(d->router_w) : nullptr, E, H, wpart, x, T,
                           reinterpret_cast<float*>(w8 + L.xn2), sms, s));
        pdl = !timed;
    }

    // 1. router logits
    const float* logits = d->router_logits;
    float* logits_rw = nullptr;
    if (!logits) {
        float* lg = logits_out ? logits_out : reinterpret_cast<float*>(w8 + L.logits);
        if (!mark()) return MOE_ERR_CUDA;
        if (!dense_router && T <= 64 && router_small_supported(H)) {
            // the many-token path without a prep kernel: this first kernel zeroes the counters
            const bool lp = path == MOE_PATH_LARGE;
            MOE_CK(launch_router_small(x, static_cast<const bf16*>(d->router_w), T, H, E, lg, nullptr, err, s, pdl,
                                       lp ? reinterpret_cast<int*>(w8 + L.counts) : nullptr,
                                       lp ? (int)counter_ints(E) : 0, lp ? reinterpret_cast<int*>(w8 + L.done) : nullptr,
                                       lp ? kStreamKMaxTiles : 0));
        } else {
            st = run_router_dense(d, x, lg, nullptr, sms, s, err, pdl);
            if (st != MOE_OK) return st;
        }
        logits = lg;
        logits_rw = lg;
        pdl = !timed;
    } else if (logits_out) {
        MOE_CK(cudaMemcpyAsync(logits_out, logits, (size_t)T * E * 4, cudaMemcpyDeviceToDevice, s));
        pdl = false;  // the next kernel follows a copy, not a kernel: no programmatic overlap
    }

    if (path == MOE_PATH_SMALL) {
        RouteTable* rt = reinterpret_cast<RouteTable*>(w8 + L.route);
        if (!mark()) return MOE_ERR_CUDA;
        const GateArgs ga = {x, static_cast<const bf16*>(d->shared_gate_w), H, rt->gate};
        MOE_CK(launch_route_small(logits, T, E, K, d->score, d->bias, d->renorm, rt, topk_w_out, topk_ids_out, s,
                                  pdl && !timed, ga));
        SmallArgs a;
        std::memset(&a, 0, sizeof(a));
        a.T = T;
        a.H = H;
        a.I = I;
        a.E = E;
        a.K = K;
        a.act = d->act;
        a.score = d->score;
        a.renorm = d->renorm;
        a.Is = Is;
        a.rt = rt;
        a.x = x;
        a.w13 = static_cast<const bf16*>(d->w13);
        a.w2 = static_cast<const bf16*>(d->w2);
        a.ws13 = static_cast<const bf16*>(d->ws13);
        a.ws2 = static_cast<const bf16*>(d->ws2);
        a.h = reinterpret_cast<bf16*>(w8 + L.h);
        a.hs = reinterpret_cast<bf16*>(w8 + L.hs);
        a.out = out;
        a.routed_scale = rscale;
        a.has_gate = d->shared_gate_w != nullptr;
        a.sh_out = sh_out;
        const std::function<bool()> mark_fn = mark;
        MOE_CK(launch_small(a, sms, s, true, timed ? &mark_fn : nullptr));
        if (!mark()) return MOE_ERR_CUDA;
        return MOE_OK;
    }

    // ---- many-token path
    float* tw = reinterpret_cast<float*>(w8 + L.topk_w);
    int32_t* tid = reinterpret_cast<int32_t*>(w8 + L.topk_ids);
    int32_t* offsets = reinterpret_cast<int32_t*>(w8 + L.offsets);
    int32_t* tiles1 = reinterpret_cast<int32_t*>(w8 + L.tiles1);
    int32_t* tiles2 = reinterpret_cast<int32_t*>(w8 + L.tiles2);
    int32_t* perm = reinterpret_cast<int32_t*>(w8 + L.perm);
    int* counts = reinterpret_cast<int*>(w8 + L.counts);
    int* cursor = counts + (E + 2);
    bf16* h = reinterpret_cast<bf16*>(w8 + L.h);
    bf16* hs = reinterpret_cast<bf16*>(w8 + L.hs);
    float* acc = reinterpret_cast<float*>(w8 + L.acc);
    float* acc_s = Is ? acc + (size_t)T * H : nullptr;
    float* gate = d->shared_gate_w ? reinterpret_cast<float*>(w8 + L.gate) : nullptr;
    const GateArgs ga = {x, static_cast<const bf16*>(d->shared_gate_w), H, gate};

    const bool chain = !timed;  // programmatic overlap between consecutive kernels
    const bool swiglu = d->act == MOE_ACT_SWIGLU;
    const int fc1_mode = swiglu ? GM_FC1_SWIGLU : GM_FC1_RELU2;
    const int bn1 = fc1_tile_rows(d), bn2 = fc2_tile_rows(d);
    const bool dyn = resolve_schedule(d) == MOE_SCHED_DYNAMIC;
    // 2. top-k (also counts the slots per expert; the counters were cleared in step 0)
    if (!mark()) return MOE_ERR_CUDA;
    RefineArgs ra = {x, static_cast<const bf16*>(d->router_w), H, logits_rw, wpart, prep_grid(E, T, sms),
                     reinterpret_cast<const float*>(w8 + L.xn2), err};
    if (dense_router && split_topk_mode(d)) {  // screen, refine, final
        int* cbase = reinterpret_cast<int*>(w8 + L.cand);
        CandList cl;
        cl.count = counts + cand_count_int(E);
        cl.row_base = cbase;
        cl.row_n = cbase + T;
        cl.row_eps = reinterpret_cast<float*>(w8 + L.roweps);
        cl.cand_row = cbase + 2 * (size_t)T;
        cl.cand_e = cl.cand_row + kCandPerRow * (size_t)T;
        cl.cand_val = reinterpret_cast<float*>(cl.cand_e + kCandPerRow * (size_t)T);
        cl.cap = (int)(kCandPerRow * (size_t)T);
        const std::function<bool()> mark_fn = mark;
        MOE_CK(launch_topk_split(logits, T, E, K, d->score, d->bias, d->renorm, tw, tid, topk_w_out, topk_ids_out,
                                 cl, ra, counts, err, sms, s, pdl && chain, timed ? &mark_fn : nullptr, ga));
    } else {
        MOE_CK(launch_topk(logits, false, T, E, K, d->score, d->bias, d->renorm, tw, tid, nullptr, topk_w_out,
                           topk_ids_out, s, pdl && chain, dense_router ? &ra : nullptr, counts, &ga));
    }
    // 3. permutation + tile tables
    PermuteArgs pa;
    std::memset(&pa, 0, sizeof(pa));
    pa.ids = tid;
    pa.M = T;
    pa.K = K;
    pa.E = E;
    pa.offsets = offsets;
    pa.perm = perm;
    pa.err = err;
    pa.has_shared = Is > 0;
    pa.bn1 = bn1;
    pa.bn2 = bn2;
    pa.nfeat1_r = cdiv(I, 128);
    pa.nfeat1_s = cdiv(Is, 128);
    pa.nfeat2_r = cdiv(H, 128);
    pa.nfeat2_s = cdiv(H, 128);
    pa.tiles1 = tiles1;
    pa.tiles2 = tiles2;
    if (!mark()) return MOE_ERR_CUDA;
    MOE_CK(launch_permute_fast(pa, counts, cursor, s, chain));

    // 4. FC1 (+ activation), zeroing acc for FC2
    const uint64_t rows1 = swiglu ? 2ull * I : (uint64_t)I;
    const uint64_t rows1s = swiglu ? 2ull * Is : (uint64_t)Is;
    GemmMaps m1;
    std::memset(&m1, 0, sizeof(m1));
    if (!map3d(&m1.a_r, d->w13, H, rows1, E, 128)) return MOE_ERR_CUDA;
    if (Is) {
        if (!map2d(&m1.a_s, d->ws13, H, rows1s, 128)) return MOE_ERR_CUDA;
    } else {
        m1.a_s = m1.a_r;
    }
    m1.b_r = m1.a_r;
    m1.b_s = m1.a_r;
    GemmArgs g1;
    std::memset(&g1, 0, sizeof(g1));
    g1.T = T;
    g1.K = K;
    g1.kdim = H;
    g1.kdim_s = H;
    g1.nfeat_r = cdiv(I, 128);
    g1.nfeat_s = cdiv(Is, 128);
    g1.feat_r = I;
    g1.feat_s = Is;
    g1.up_r = I;
    g1.up_s = Is;
    g1.E = E;
    g1.has_shared = Is > 0;
    g1.offsets = offsets;
    g1.tiles = tiles1;
    g1.perm = perm;
    g1.topk_w = tw;
    g1.xsrc = x;
    g1.h = h;
    g1.hs = hs;
    g1.trace = d->trace ? d->trace + (size_t)MOE_TRACE_FC1 * MOE_TRACE_MAX_CTAS * MOE_TRACE_FIELDS : nullptr;
    g1.zero_ptr = acc;
    g1.zero_n = (size_t)T * H * (Is ? 2 : 1);
    // Upper bound of a grouped GEMM's tiles: at most min(E, T*K) experts have rows, and each
    // expert's token tiles add at most one beyond its share of T*K / bn; plus the shared group.
    auto max_tiles = [&](int bn, int nf_r, int nf_s) {
        const long long TK = (long long)T * K;
        return (long long)nf_r * (std::min<long long>(E, TK) + TK / bn) + (long long)nf_s * cdiv(T, bn);
    };
    g1.streamk_max = gemm_streamk_max(fc1_mode, bn1, sms, max_tiles(bn1, g1.nfeat_r, Is ? g1.nfeat_s : 0));
    g1.skp = reinterpret_cast<float*>(w8 + L.skp);
    g1.done = reinterpret_cast<int*>(w8 + L.done);
    g1.dyn_ctr = dyn ? counts + dyn_count_int(E, 0) : nullptr;
    g1.err = err;
    if (!mark()) return MOE_ERR_CUDA;
    MOE_CK(launch_gemm(fc1_mode, bn1, g1, m1, sms, s, chain));

    // 5. FC2 + weighted scatter-add (shared expert -> ys)
    GemmMaps m2;
    std::memset(&m2, 0, sizeof(m2));
    if (!map3d(&m2.a_r, d->w2, I, H, E, 128) || !map2d(&m2.b_r, h, I, (uint64_t)T * K, kFc2BoxRows)) return MOE_ERR_CUDA;
    if (Is) {
        if (!map2d(&m2.a_s, d->ws2, Is, H, 128) || !map2d(&m2.b_s, hs, Is, T, kFc2BoxRows)) return MOE_ERR_CUDA;
    } else {
        m2.a_s = m2.a_r;
        m2.b_s = m2.b_r;
    }
    GemmArgs g2 = g1;
    g2.kdim = I;
    g2.kdim_s = Is;
    g2.nfeat_r = cdiv(H, 128);
    g2.nfeat_s = cdiv(H, 128);
    g2.feat_r = H;
    g2.feat_s = H;
    g2.tiles = tiles2;
    g2.trace = d->trace ? d->trace + (size_t)MOE_TRACE_FC2 * MOE_TRACE_MAX_CTAS * MOE_TRACE_FIELDS : nullptr;
    g2.acc = acc;
    g2.acc_s = acc_s;
    g2.sgate = gate;
    g2.zero_ptr = nullptr;
    g2.zero_n = 0;
    g2.streamk_max = gemm_streamk_max(GM_FC2, bn2, sms, max_tiles(bn2, g2.nfeat_r, Is ? g2.nfeat_s : 0));
    g2.skp = nullptr;
    g2.done = nullptr;
    g2.dyn_ctr = dyn ? counts + dyn_count_int(E, 1) : nullptr;

    if (!mark()) return MOE_ERR_CUDA;
    MOE_CK(launch_gemm(GM_FC2, bn2, g2, m2, sms, s, chain));

    // 6. finalize
    if (!mark()) return MOE_ERR_CUDA;
    MOE_CK(launch_finalize(acc, acc_s, sh_out, out, (size_t)T * H, rscale, sms, s, chain));
    if (!mark()) return MOE_ERR_CUDA;
    return MOE_OK;
}

moe_status_t moe_fused_forward(const moe_layer_desc* d, const void* x, void* out, float* topk_w_out,
                               int32_t* topk_ids_out, float* logits_out, void* ws, size_t ws_bytes, void* stream) {
    return fused_forward_impl(d, x, out, topk_w_out, topk_ids_out, logits_out, ws, ws_bytes, stream, nullptr, 0);
}

moe_status_t moe_fused_forward_timed(const moe_layer_desc* d, const void* x, void* out, float* topk_w_out,
                                     int32_t* topk_ids_out, float* logits_out, void* ws, size_t ws_bytes,
                                     void* stream, void* const* events, int n_events) {
    if (!events) return MOE_ERR_INVALID_ARG;
    return fused_forward_impl(d, x, out, topk_w_out, topk_ids_out, logits_out, ws, ws_bytes, stream, events,
                              n_events);
}

moe_status_t moe_get_error(void* ws, int* code, void* stream) {
    if (!ws || !code) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    int* err = &static_cast<WsHeader*>(ws)->err;
    int v = 0;
    if (cudaMemcpyAsync(&v, err, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemsetAsync(err, 0, sizeof(int), s) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
    *code = v;
    return v ? MOE_ERR_DEVICE : MOE_OK;
}

}  // extern "C"
