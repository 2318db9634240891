// router.cu -- router logits for few tokens (weight streaming) and the warp-per-row
// router top-k kernel behind moe_router_topk and the large-token path.
#include "kernels.cuh"
#include "router.cuh"

namespace moe {

// ---------------------------------------------------------------- top-k, one warp per row
// With `refine` (logits from the tensor-core router, FP32 accumulation in the MMA's own
// order): a first selection on those logits; then every expert whose key lies within
// `kRefineWindow` (relative) of the K-th key -- the selected ones included -- gets its
// logit recomputed as an FP64 dot product rounded once to FP32, written back, and the
// selection and weights are redone.  An expert outside the window cannot enter the top
// K as long as the tensor-core logit error stays below half the window (it is ~1e-6
// absolute on these workloads against a window of 2e-3), so ids and weights follow the
// correctly rounded logits.
static constexpr float kRefineWindow = 2e-3f;

template <int V>
__device__ __forceinline__ void refine_row(float (&l)[V], int row, int E, int K, int score, const float* bias,
                                           int renorm, int lane, const bf16* x, const bf16* wr, int H,
                                           float* logits_rw) {
    int id;
    float w, lg;
    warp_topk_row<V>(l, E, K, score, bias, renorm, lane, id, w, lg);
    // K-th key of the first selection
    const int idK = __shfl_sync(0xffffffffu, id, K - 1);
    const float lK = __shfl_sync(0xffffffffu, lg, K - 1);
    float kK = (score == MOE_SCORE_SIGMOID) ? sigmoid_f32_rn(lK) : lK;
    if (bias) kK = __fadd_rn(kK, bias[idK]);
    const float win = kRefineWindow * fmaxf(1.0f, fabsf(kK)) * (score == MOE_SCORE_SIGMOID ? 0.25f : 1.0f);
    const bf16* xr = x + (size_t)row * H;
    const int nch = H >> 3;
#pragma unroll
    for (int c = 0; c < V; ++c) {
        const int e = lane + 32 * c;
        bool cand = false;
        if (e < E) {
            float k = (score == MOE_SCORE_SIGMOID) ? sigmoid_f32_rn(l[c]) : l[c];
            if (bias) k = __fadd_rn(k, bias[e]);
            cand = !(k < kK - win);  // also true for NaN
        }
        unsigned m = __ballot_sync(0xffffffffu, cand);
        while (m) {
            const int src = __ffs(m) - 1;
            m &= m - 1;
            const int ee = src + 32 * c;
            const bf16* wrow = wr + (size_t)ee * H;
            // four independent partial sums keep four 16-byte chunks of the row in flight
            double acc0 = 0.0, acc1 = 0.0, acc2 = 0.0, acc3 = 0.0;
            int q = lane;
            for (; q + 96 < nch; q += 128) {
                const uint4 w0 = ld_nc16(wrow + (size_t)q * 8), w1 = ld_nc16(wrow + (size_t)(q + 32) * 8);
                const uint4 w2 = ld_nc16(wrow + (size_t)(q + 64) * 8), w3 = ld_nc16(wrow + (size_t)(q + 96) * 8);
                const uint4 x0 = ld_nc16(xr + (size_t)q * 8), x1 = ld_nc16(xr + (size_t)(q + 32) * 8);
                const uint4 x2 = ld_nc16(xr + (size_t)(q + 64) * 8), x3 = ld_nc16(xr + (size_t)(q + 96) * 8);
                acc0 = dot8_f64(x0, w0, acc0);
                acc1 = dot8_f64(x1, w1, acc1);
                acc2 = dot8_f64(x2, w2, acc2);
                acc3 = dot8_f64(x3, w3, acc3);
            }
            for (; q < nch; q += 32) acc0 = dot8_f64(ld_nc16(xr + (size_t)q * 8), ld_nc16(wrow + (size_t)q * 8), acc0);
            const float exact = __double2float_rn(warp_sum_f64((acc0 + acc1) + (acc2 + acc3)));
            if (lane == src) {
                l[c] = exact;
                if (logits_rw) logits_rw[(size_t)row * E + ee] = exact;
            }
        }
    }
}

template <int V, bool BF16_IN, bool REFINE>
__global__ void __launch_bounds__(256) topk_kernel(const void* __restrict__ logits, int M, int E, int K, int score,
                                                   const float* __restrict__ bias, int renorm,
                                                   float* __restrict__ topk_w, int32_t* __restrict__ topk_ids,
                                                   int32_t* __restrict__ src_idx, float* __restrict__ w_copy,
                                                   int32_t* __restrict__ id_copy, const bf16* __restrict__ x,
                                                   const bf16* __restrict__ wr, int H, float* logits_rw,
                                                   int* __restrict__ counts) {
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (row < M) {
        float l[V];
        if (BF16_IN)
            load_row_bf16<V>(static_cast<const uint16_t*>(logits) + (size_t)row * E, E, lane, l);
        else
            load_row_f32<V>(static_cast<const float*>(logits) + (size_t)row * E, E, lane, l);
        if (REFINE) refine_row<V>(l, row, E, K, score, bias, renorm, lane, x, wr, H, logits_rw);
        int id;
        float w, lg;
        warp_topk_row<V>(l, E, K, score, bias, renorm, lane, id, w, lg);
        if (lane < K) {
            const size_t o = (size_t)row * K + lane;
            topk_w[o] = w;
            topk_ids[o] = id;
            if (src_idx) src_idx[o] = lane * M + row;
            if (w_copy) w_copy[o] = w;
            if (id_copy) id_copy[o] = id;
            if (counts) atomicAdd(counts + id, 1);
        }
    }
    pdl_trigger();
}

cudaError_t launch_topk(const void* logits, bool bf16_in, int M, int E, int K, int score, const float* bias,
                        int renorm, float* topk_w, int32_t* topk_ids, int32_t* src_idx, float* w_copy,
                        int32_t* id_copy, cudaStream_t s, bool pdl, const RefineArgs* refine, int* counts) {
    const int rows_per_block = 8;
    dim3 grid(cdiv(M, rows_per_block)), block(32 * rows_per_block);
    const int v = topk_v(E);
    const bf16* x = refine ? refine->x : nullptr;
    const bf16* wr = refine ? refine->wr : nullptr;
    const int H = refine ? refine->H : 0;
    float* lrw = refine ? refine->logits_rw : nullptr;
#define MOE_L(VV)                                                                                              \
    if (v == VV) {                                                                                             \
        if (refine)                                                                                            \
            return launch_k(topk_kernel<VV, false, true>, grid, block, 0, s, pdl, logits, M, E, K, score, bias, \
                            renorm, topk_w, topk_ids, src_idx, w_copy, id_copy, x, wr, H, lrw, counts);        \
        return bf16_in ? launch_k(topk_kernel<VV, true, false>, grid, block, 0, s, pdl, logits, M, E, K, score, \
                                  bias, renorm, topk_w, topk_ids, src_idx, w_copy, id_copy, x, wr, H, lrw, counts) \
                       : launch_k(topk_kernel<VV, false, false>, grid, block, 0, s, pdl, logits, M, E, K, score, \
                                  bias, renorm, topk_w, topk_ids, src_idx, w_copy, id_copy, x, wr, H, lrw, counts); \
    }
    MOE_L(1) MOE_L(2) MOE_L(4) MOE_L(8) MOE_L(16) MOE_L(32)
#undef MOE_L
    return cudaErrorInvalidValue;
}

// ---------------------------------------------------------------- router logits, few tokens
// l[t, e] = x[t,:] . Wr[e,:].  One warp per expert row: the lanes stream the row in
// 16-byte chunks once (HBM), and dot each chunk with the matching chunk of every token
// (x is tiny and stays in L1/L2).  The accumulation is FP64 (BF16 products are exact in
// double), so the FP32 logit is the correctly rounded dot product except when the exact
// value lies within ~1e-16 of an FP32 rounding boundary.
template <int VH, int TT>
__global__ void __launch_bounds__(128) router_logits_small(const bf16* __restrict__ x, const bf16* __restrict__ wr,
                                                           int T, int H, int E, float* __restrict__ logits,
                                                           float* __restrict__ logits_copy) {
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int e = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (e < E) {
        const int nch = H >> 3;  // 16-byte chunks per row
        const bf16* wrow = wr + (size_t)e * H;
        uint4 w[VH];  // the whole row is loaded at once: one memory latency per row
#pragma unroll
        for (int j = 0; j < VH; ++j) {
            const int c = lane + 32 * j;
            w[j] = (c < nch) ? ld_stream16(wrow + (size_t)c * 8) : make_uint4(0u, 0u, 0u, 0u);
        }
        for (int t0 = 0; t0 < T; t0 += TT) {
            double acc[TT];
#pragma unroll
            for (int i = 0; i < TT; ++i) acc[i] = 0.0;
#pragma unroll
            for (int j = 0; j < VH; ++j) {
                const int c = lane + 32 * j;
                if (c < nch) {
#pragma unroll
                    for (int i = 0; i < TT; ++i)
                        if (t0 + i < T) acc[i] = dot8_f64(w[j], ld_nc16(x + (size_t)(t0 + i) * H + (size_t)c * 8), acc[i]);
                }
            }
#pragma unroll
            for (int i = 0; i < TT; ++i) {
                const float v = __double2float_rn(warp_sum_f64(acc[i]));
                if (lane == 0 && t0 + i < T) {
                    logits[(size_t)(t0 + i) * E + e] = v;
                    if (logits_copy) logits_copy[(size_t)(t0 + i) * E + e] = v;
                }
            }
        }
    }
    pdl_trigger();
}

bool router_small_supported(int H) { return (H >> 3) <= 32 * 16; }

cudaError_t launch_router_small(const bf16* x, const bf16* wr, int T, int H, int E, float* logits,
                                float* logits_copy, cudaStream_t s, bool pdl) {
    dim3 grid(cdiv(E, 4)), block(128);
    const int need = cdiv(H >> 3, 32);
#define MOE_R(VV)                                                                                               \
    if (need <= VV) {                                                                                           \
        if (T <= 2)                                                                                             \
            return launch_k(router_logits_small<VV, 2>, grid, block, 0, s, pdl, x, wr, T, H, E, logits, logits_copy); \
        if (T <= 4)                                                                                             \
            return launch_k(router_logits_small<VV, 4>, grid, block, 0, s, pdl, x, wr, T, H, E, logits, logits_copy); \
        return launch_k(router_logits_small<VV, 8>, grid, block, 0, s, pdl, x, wr, T, H, E, logits, logits_copy);     \
    }
    MOE_R(4) MOE_R(8) MOE_R(12) MOE_R(16)
#undef MOE_R
    return cudaErrorInvalidValue;
}

}  // namespace moe
