// kernels.cuh -- launch interfaces between the host API (api.cu) and the kernels.
#pragma once
#include <algorithm>
#include <functional>

#include "moe_internal.cuh"

namespace moe {

// Launch with the programmatic-dependent-launch attribute when `pdl` is set: the kernel
// may start while the previous kernel in the stream drains; every kernel calls
// griddepcontrol.wait before it reads what the previous one wrote.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl,
                     Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------- router
// FP64 re-evaluation of the candidate logits after the tensor-core router (see router.cu).
struct RefineArgs {
    const bf16* x;       // [M, H]
    const bf16* wr;      // [E, H]
    int H;
    float* logits_rw;    // refined logits are written back here (the logits buffer)
    const float* wpart;  // [nwpart] per-CTA upper bounds of max_e |Wr[e]|_2^2 (prep kernel)
    int nwpart;
    const float* xn2;    // [M] upper bounds of |x_t|_2^2 (prep kernel)
    int* err;            // device error word (MOE_DEVERR_ROUTER_BOUND)
};
// Shared-expert gate of each token, computed by the routing kernels (one exact dot
// product per row): out[t] = sigmoid_f32(x[t] . w), w == null = no gate.
struct GateArgs {
    const bf16* x;  // [M, H]
    const bf16* w;  // [H] or null
    int H;
    float* out;     // [M]
};
cudaError_t launch_topk(const void* logits, bool bf16_in, int M, int E, int K, int score, const float* bias,
                        int renorm, float* topk_w, int32_t* topk_ids, int32_t* src_idx, float* w_copy,
                        int32_t* id_copy, cudaStream_t s, bool pdl, const RefineArgs* refine = nullptr,
                        int* counts = nullptr, const GateArgs* gate = nullptr);
// Candidate list of the three-kernel top-k after the tensor-core router.
struct CandList {
    int* count;       // [1] candidates appended so far (zero on entry)
    int* row_base;    // [M] first list entry of each row
    int* row_n;       // [M] candidates of each row
    int* cand_row;    // [cap]
    int* cand_e;      // [cap]
    float* cand_val;  // [cap] exact logits
    float* row_eps;   // [M] error bound of each row's tensor-core logits
    int cap;
};
// screen, refine and final kernels; `mark` (optional) records a timing event between them.
cudaError_t launch_topk_split(const float* logits, int M, int E, int K, int score, const float* bias, int renorm,
                              float* topk_w, int32_t* topk_ids, float* w_copy, int32_t* id_copy, const CandList& cl,
                              const RefineArgs& ra, int* counts, int* err, int num_sms, cudaStream_t s, bool pdl,
                              const std::function<bool()>* mark, const GateArgs& gate);
bool router_small_supported(int H);
// zero_ints / zero_ints2 (optional, n_zero / n_zero2 ints): counters the kernel zeroes as a
// call's first kernel.
cudaError_t launch_router_small(const bf16* x, const bf16* wr, int T, int H, int E, float* logits,
                                float* logits_copy, int* err, cudaStream_t s, bool pdl, int* zero_ints = nullptr,
                                int n_zero = 0, int* zero_ints2 = nullptr, int n_zero2 = 0);

// ---------------------------------------------------------------- few-token path
static constexpr int kSmallMaxT = 16;
static constexpr int kSmallMaxSlots = kSmallMaxT * MOE_MAX_TOPK;
// Routing of the few-token path, built once by route_small_kernel: the distinct experts
// in ascending order (ulist), and for each the slots k*T + t it serves
// (utok[uoff[u] .. uoff[u+1])), plus every slot's expert and weight (index t*K + k).
struct RouteTable {
    int U;
    int pad[31];
    int ulist[kSmallMaxSlots];
    int uoff[kSmallMaxSlots + 1];
    int utok[kSmallMaxSlots];
    int ids[kSmallMaxSlots];
    float w[kSmallMaxSlots];
    float gate[kSmallMaxT];  // shared-expert gate of each token (when the layer has one)
};
cudaError_t launch_route_small(const float* logits, int T, int E, int K, int score, const float* bias, int renorm,
                               RouteTable* rt, float* w_out, int32_t* id_out, cudaStream_t s, bool pdl,
                               const GateArgs& gate);
struct SmallArgs {
    int T, H, I, E, K, act, score, renorm, Is;
    const RouteTable* rt;
    const bf16* x;
    const bf16* w13;
    const bf16* w2;
    const bf16* ws13;
    const bf16* ws2;
    bf16* h;           // [T*K, I], row = slot k*T + t
    bf16* hs;          // [T, Is]
    bf16* out;         // [T, H] (may equal sh_out)
    float routed_scale;  // multiplies the routed sum before its BF16 rounding
    int has_gate;        // the shared output is multiplied by rt->gate[t]
    const bf16* sh_out;  // [T, H] caller-computed shared output (Is == 0), or null
};
bool small_path_supported(int T, int H, int I, int Is);
// `mark` (optional) records a timing event before each of the two streaming kernels;
// when it is given the kernels are launched without programmatic overlap.
cudaError_t launch_small(const SmallArgs& a, int num_sms, cudaStream_t s, bool pdl_first,
                         const std::function<bool()>* mark);

// First kernel of a many-token call: zeroes the call's counters (n and n2 ints) and, when wr is
// given, writes per-CTA upper bounds of max_e |wr[e]|_2^2 into wpart[prep_grid(E, T, sms)]
// and upper bounds of |x_t|_2^2 into xn2[T] (the bound on the tensor-core router's error).
int prep_grid(int E, int T, int num_sms);
cudaError_t launch_prep(int* counters, int n, int* counters2, int n2, const bf16* wr, int E, int H, float* wpart,
                        const bf16* x, int T, float* xn2, int num_sms, cudaStream_t s);

// ---------------------------------------------------------------- permutation
// Tile bookkeeping that the permute kernel writes for the grouped GEMMs (group g < E is
// routed expert g; g == E is the shared expert when present, with T rows).
struct PermuteArgs {
    const int32_t* ids;  // [M, K]
    int M, K, E;
    int32_t* offsets;    // [E + 1]
    int32_t* perm;       // [M*K]
    int32_t* inv;        // [M*K] or null
    int* err;
    // grouped-GEMM tile tables (null when not wanted)
    int has_shared;      // adds group E with M rows
    int bn1, bn2;        // token rows per tile of the FC1 / FC2 GEMMs
    int nfeat1_r, nfeat1_s, nfeat2_r, nfeat2_s;
    int32_t* tiles1;     // [G + 1] exclusive prefix of FC1 tiles over groups
    int32_t* tiles2;     // [G + 1] exclusive prefix of FC2 tiles over groups
};
size_t permute_smem_bytes(int E);
cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t s, bool pdl);
// Fused-path permutation: the per-expert counts were accumulated by the top-k kernel.
// Each CTA ranks its slots per expert in shared memory and reserves one contiguous range
// per expert with a single atomic on the expert's cursor (order within an expert is not
// fixed).  `cursor` [E] must be zero on entry.
cudaError_t launch_permute_fast(const PermuteArgs& a, const int* counts, int* cursor, cudaStream_t s, bool pdl);

// ---------------------------------------------------------------- grouped tcgen05 GEMM
enum GemmMode { GM_FC1_SWIGLU = 0, GM_FC1_RELU2 = 1, GM_FC2 = 2, GM_DENSE = 3 };
// Token rows per tile of the dense router GEMM (E is small, so narrow token tiles give the
// grid its width; measured: 256-token tiles with split-K and FP32 atomics into the logits
// were 3x slower).  The grouped FC1 / FC2 GEMMs take gemm_token_tile(mode, T, K, E).
static constexpr int kDenseTokenTile = 64;
struct GemmArgs {
    int T, K;            // tokens and top-k (slot decode of perm entries)
    int kdim;            // reduction length (H for FC1 / router, I or I_s for FC2)
    int kdim_s;          // reduction length of the shared group
    int nfeat_r, nfeat_s;  // 128-row feature tiles per routed / shared group
    int feat_r, feat_s;    // valid output features per routed / shared group
    int up_r, up_s;        // SwiGLU: row offset of the up half (I, I_s)
    int E;               // routed groups; group E = shared (if has_shared)
    int has_shared;
    int dense;           // GM_DENSE: one group of T rows, tiles = nfeat_r * ceil(T / kDenseTokenTile)
    const int32_t* offsets;  // [E + 1] permuted row offsets of the routed groups
    const int32_t* tiles;    // [G + 1] tile prefix (group-major)
    const int32_t* perm;     // [T*K] source slot indices k*T + t
    const float* topk_w;     // [T, K]
    const bf16* xsrc;        // FC1 gather source x [T, H]
    bf16* h;                 // FC1 routed out [T*K, I]
    bf16* hs;                // FC1 shared out [T, I_s]
    float* acc;              // FC2 routed out [T, H] (FP32 red.add)
    float* acc_s;            // FC2 shared-expert out [T, H] (FP32 red.add)
    float* logits;           // GM_DENSE out [T, E]
    float* logits_copy;      // GM_DENSE optional second output
    float* zero_ptr;         // FC1: buffer zeroed by the epilogue warps before their tiles
    size_t zero_n;           //      (floats, multiple of 4)
    const float* sgate;      // FC2: shared-expert gate per token (acc_s += gate[t] * y), or null
    unsigned long long* trace;  // this kernel's phase-trace block ([grid][MOE_TRACE_FIELDS]) or null
    int streamk_max;         // stream-K when the call has fewer tiles than this (0: never)
    float* skp;              // FC1 stream-K partial sums, one slot per CTA ([kNA][BN][128] FP32)
    int* done;               // FC1 stream-K per-tile counters (zero on entry, >= streamk_max of them)
    int* dyn_ctr;            // dynamic tile schedule: the next-tile counter (zero on entry), or null
    int* err;
};
struct GemmMaps {
    CUtensorMap a_r;  // routed weights (3D [E][rows][kdim]) or dense A (2D)
    CUtensorMap a_s;  // shared weights (2D)
    CUtensorMap b_r;  // FC2: h [T*K, I]; DENSE: x [T, H] (16-row boxes)
    CUtensorMap b_s;  // FC2: hs [T, I_s]
};
// Token rows per tile of a grouped GEMM for a call over T tokens, top-k K and E experts:
// 32 when T <= 32 (no expert can have more rows), else by the average rows per expert
// (FC1: 64 up to 48 rows, else 128, and 256 above 96 for ReLU^2; FC2: 128 up to 64
// rows, 192 up to 150, else 256).  Narrow tiles leave shared memory for a deeper
// weight ring.  The permute kernel's tile tables must use the same value as the launch.
int gemm_token_tile(int mode, int T, int K, int E);
// Rows per TMA box of FC2's h / hs tensor maps (the kernel's copies use the same box).
constexpr int kFc2BoxRows = 32;
cudaError_t launch_gemm(int mode, int bn, const GemmArgs& a, const GemmMaps& m, int grid, cudaStream_t s, bool pdl);

// Stream-K limits: FC1 and FC2 run stream-K while a call has fewer tiles than
// kStreamKWaves waves of the grid; FC1 only with token tiles of at most 64 rows (its
// partial-sum slots) and at most kStreamKMaxTiles tiles (its counters).
static constexpr int kStreamKWaves = 8;
static constexpr int kStreamKMaxTiles = 1024;
static constexpr int kStreamKMaxBN = 64;
// Bytes of FC1's stream-K partial-sum slots for `grid` CTAs (0 when FC1 cannot use it).
size_t fc1_streamk_bytes(int bn, bool swiglu, int grid);
// Stream-K tile limit for a call whose tile count is at most max_tiles (0: whole tiles).
int gemm_streamk_max(int mode, int bn, int grid, long long max_tiles);

// finalize: out = bf16(bf16(scale * acc) + shared) with shared = bf16(acc_s) (internal
// shared expert) or sh_out (caller's), or bf16(scale * acc) without one.  out may equal
// sh_out (each element is read before it is written, by the same thread).
cudaError_t launch_finalize(const float* acc, const float* acc_s, const bf16* sh_out, bf16* out, size_t n,
                            float scale, int num_sms, cudaStream_t s, bool pdl);

// Driver entry point for tensor-map encoding (resolved once through the runtime).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn get_encode_tiled();

}  // namespace moe
