// router.cu -- router logits for few tokens (weight streaming) and the warp-per-row
// router top-k kernel behind moe_router_topk and the large-token path.
#include "kernels.cuh"
#include "router.cuh"

namespace moe {

// ---------------------------------------------------------------- top-k, one warp per row
template <int V, bool BF16_IN>
__global__ void __launch_bounds__(256) topk_kernel(const void* __restrict__ logits, int M, int E, int K, int score,
                                                   const float* __restrict__ bias, int renorm,
                                                   float* __restrict__ topk_w, int32_t* __restrict__ topk_ids,
                                                   int32_t* __restrict__ src_idx, float* __restrict__ w_copy,
                                                   int32_t* __restrict__ id_copy) {
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (row < M) {
        float l[V];
        if (BF16_IN)
            load_row_bf16<V>(static_cast<const uint16_t*>(logits) + (size_t)row * E, E, lane, l);
        else
            load_row_f32<V>(static_cast<const float*>(logits) + (size_t)row * E, E, lane, l);
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
        }
    }
    pdl_trigger();
}

cudaError_t launch_topk(const void* logits, bool bf16_in, int M, int E, int K, int score, const float* bias,
                        int renorm, float* topk_w, int32_t* topk_ids, int32_t* src_idx, float* w_copy,
                        int32_t* id_copy, cudaStream_t s, bool pdl) {
    const int rows_per_block = 8;
    dim3 grid(cdiv(M, rows_per_block)), block(32 * rows_per_block);
    const int v = topk_v(E);
#define MOE_L(VV)                                                                                                \
    if (v == VV)                                                                                                 \
        return bf16_in ? launch_k(topk_kernel<VV, true>, grid, block, 0, s, pdl, logits, M, E, K, score, bias, \
                                  renorm, topk_w, topk_ids, src_idx, w_copy, id_copy)                            \
                       : launch_k(topk_kernel<VV, false>, grid, block, 0, s, pdl, logits, M, E, K, score, bias, \
                                  renorm, topk_w, topk_ids, src_idx, w_copy, id_copy);
    MOE_L(1) MOE_L(2) MOE_L(4) MOE_L(8) MOE_L(16) MOE_L(32)
#undef MOE_L
    return cudaErrorInvalidValue;
}

// ---------------------------------------------------------------- router logits, few tokens
// l[t, e] = x[t,:] . Wr[e,:].  One warp per expert row: the lanes stream the row in
// 16-byte chunks once (HBM), and dot each chunk with the matching chunk of every token
// (x is tiny and stays in L1/L2).  FP32 accumulation, XOR-tree reduction.
template <int TT>
__global__ void __launch_bounds__(128) router_logits_small(const bf16* __restrict__ x, const bf16* __restrict__ wr,
                                                           int T, int H, int E, float* __restrict__ logits,
                                                           float* __restrict__ logits_copy) {
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int e = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (e < E) {
        const int nch = H >> 3;  // 16-byte chunks per row
        const bf16* wrow = wr + (size_t)e * H;
        for (int t0 = 0; t0 < T; t0 += TT) {
            float acc[TT];
#pragma unroll
            for (int j = 0; j < TT; ++j) acc[j] = 0.0f;
            for (int c = lane; c < nch; c += 32) {
                const uint4 w = ld_stream16(wrow + (size_t)c * 8);
#pragma unroll
                for (int j = 0; j < TT; ++j)
                    if (t0 + j < T) acc[j] = dot8(w, ld_nc16(x + (size_t)(t0 + j) * H + (size_t)c * 8), acc[j]);
            }
#pragma unroll
            for (int j = 0; j < TT; ++j) {
                const float v = warp_sum(acc[j]);
                if (lane == 0 && t0 + j < T) {
                    logits[(size_t)(t0 + j) * E + e] = v;
                    if (logits_copy) logits_copy[(size_t)(t0 + j) * E + e] = v;
                }
            }
        }
    }
    pdl_trigger();
}

cudaError_t launch_router_small(const bf16* x, const bf16* wr, int T, int H, int E, float* logits,
                                float* logits_copy, cudaStream_t s, bool pdl) {
    dim3 grid(cdiv(E, 4)), block(128);
    if (T <= 4) return launch_k(router_logits_small<4>, grid, block, 0, s, pdl, x, wr, T, H, E, logits, logits_copy);
    if (T <= 8) return launch_k(router_logits_small<8>, grid, block, 0, s, pdl, x, wr, T, H, E, logits, logits_copy);
    return launch_k(router_logits_small<16>, grid, block, 0, s, pdl, x, wr, T, H, E, logits, logits_copy);
}

}  // namespace moe
