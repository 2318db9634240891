// router.cuh -- warp-level router top-k of one row, shared by the standalone top-k kernel
// and the fused small-token kernels.
//
// Contract ("Laguna exact M=8 BF16-input router top-k preregistration", section
// "Question and arithmetic contract"): logits widened exactly to FP32; sigmoid score
// s = sigmoid(l) in FP32 (here: correctly rounded from an FP64 evaluation); key = s + b in
// FP32 with the correction bias used for selection only; top K by (key desc, id asc);
// weights renormalise the unbiased scores.  Softmax routing keys on the logit.
//
// Layout: lane l of the warp owns experts e = l + 32 c, c = 0..V-1 (coalesced loads of
// the row).  Each of the K rounds takes every lane's best remaining (key, id) and reduces
// it across the warp with XOR shuffles 16, 8, 4, 2, 1 under the total order (key desc,
// id asc), so every lane ends with the same winner; the owner drops it.  Lane k keeps
// slot k.
#pragma once
#include "moe_internal.cuh"

namespace moe {

__device__ __forceinline__ float sigmoid_f32_rn(float l) {
    return __double2float_rn(1.0 / (1.0 + exp(-(double)l)));
}

__device__ __forceinline__ bool key_better(float ka, int ia, float kb, int ib) {
    return ka > kb || (ka == kb && ia < ib);
}

// l[c] = logit of expert lane + 32c (any value for e >= E).  Outputs valid on lanes k < K:
// id of slot k, its FP32 weight and its FP32 logit.
template <int V>
__device__ __forceinline__ void warp_topk_row(const float (&l)[V], int E, int K, int score, const float* bias,
                                              int renorm, int lane, int& out_id, float& out_w, float& out_l) {
    const float NEG_INF = __int_as_float(0xff800000);
    float key[V];
    uint32_t avail = 0;
    float lmax = NEG_INF;
#pragma unroll
    for (int c = 0; c < V; ++c) {
        const int e = lane + 32 * c;
        key[c] = NEG_INF;
        if (e < E) {
            float lv = l[c];
            float k;
            if (score == MOE_SCORE_SIGMOID) {
                float s = sigmoid_f32_rn(lv);
                k = bias ? __fadd_rn(s, bias[e]) : s;
            } else {
                k = bias ? __fadd_rn(lv, bias[e]) : lv;
            }
            key[c] = (k != k) ? NEG_INF : k;  // NaN keys are selected last
            avail |= 1u << c;
            if (lv == lv) lmax = fmaxf(lmax, lv);
        }
    }
    out_id = 0;
    out_l = 0.0f;
    for (int k = 0; k < K; ++k) {
        float bk = NEG_INF;
        int bi = 0x7fffffff;
#pragma unroll
        for (int c = 0; c < V; ++c) {
            if ((avail >> c) & 1u) {
                const int e = lane + 32 * c;
                if (key_better(key[c], e, bk, bi)) {
                    bk = key[c];
                    bi = e;
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            float ok = __shfl_xor_sync(0xffffffffu, bk, o);
            int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (key_better(ok, oi, bk, bi)) {
                bk = ok;
                bi = oi;
            }
        }
        const int owner = bi & 31, cw = bi >> 5;
        float sel = l[0];
#pragma unroll
        for (int c = 1; c < V; ++c)
            if (c == cw) sel = l[c];
        sel = __shfl_sync(0xffffffffu, sel, owner);
        if (lane == owner) avail &= ~(1u << cw);
        if (lane == k) {
            out_id = bi;
            out_l = sel;
        }
    }
    // weights
    if (score == MOE_SCORE_SIGMOID) {
        const float s = (lane < K) ? sigmoid_f32_rn(out_l) : 0.0f;
        double sum = 0.0;
        for (int k = 0; k < K; ++k) sum += (double)__shfl_sync(0xffffffffu, s, k);
        out_w = renorm ? __double2float_rn((double)s / sum) : s;
    } else {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
        const double ex = (lane < K) ? exp((double)out_l - (double)lmax) : 0.0;
        double sum = 0.0;
        if (renorm) {
            for (int k = 0; k < K; ++k) sum += __shfl_sync(0xffffffffu, ex, k);
        } else {
            double part = 0.0;
#pragma unroll
            for (int c = 0; c < V; ++c)
                if (lane + 32 * c < E) part += exp((double)l[c] - (double)lmax);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
            sum = part;
        }
        out_w = __double2float_rn(ex / sum);
    }
}

// Load one row of FP32 logits in the lane-strided layout.
template <int V>
__device__ __forceinline__ void load_row_f32(const float* row, int E, int lane, float (&l)[V]) {
#pragma unroll
    for (int c = 0; c < V; ++c) {
        const int e = lane + 32 * c;
        l[c] = (e < E) ? row[e] : 0.0f;
    }
}
template <int V>
__device__ __forceinline__ void load_row_bf16(const uint16_t* row, int E, int lane, float (&l)[V]) {
#pragma unroll
    for (int c = 0; c < V; ++c) {
        const int e = lane + 32 * c;
        l[c] = (e < E) ? __uint_as_float((uint32_t)row[e] << 16) : 0.0f;
    }
}

// Dispatch helper: V = ceil(E / 32) rounded up to a power of two (1..32).
__host__ __device__ inline int topk_v(int E) {
    int v = (E + 31) / 32;
    int p = 1;
    while (p < v) p <<= 1;
    return p;
}

// Top-k of one FP32 row with runtime E (warp-uniform dispatch on V).
__device__ __forceinline__ void warp_topk_f32(const float* row, int E, int K, int score, const float* bias,
                                              int renorm, int lane, int& id, float& w, float& lg) {
#define MOE_TOPK_CASE(VV)                                               \
    case VV: {                                                          \
        float l[VV];                                                    \
        load_row_f32<VV>(row, E, lane, l);                              \
        warp_topk_row<VV>(l, E, K, score, bias, renorm, lane, id, w, lg); \
    } break;
    switch (topk_v(E)) {
        MOE_TOPK_CASE(1)
        MOE_TOPK_CASE(2)
        MOE_TOPK_CASE(4)
        MOE_TOPK_CASE(8)
        MOE_TOPK_CASE(16)
        default:
        MOE_TOPK_CASE(32)
    }
#undef MOE_TOPK_CASE
}

}  // namespace moe
