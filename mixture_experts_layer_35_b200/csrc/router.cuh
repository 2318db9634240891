// router.cuh -- warp-level router top-k of one row, shared by every routing kernel.
//
// Contract ("Laguna exact M=8 BF16-input router top-k preregistration", section
// "Question and arithmetic contract"): logits widened exactly to FP32; sigmoid score
// s = sigmoid(l) in FP32 (correctly rounded); key = s + b in FP32 with the correction
// bias used for selection only; top K by (key desc, id asc); weights renormalise the
// unbiased scores.  Softmax routing keys on the logit.
//
// Layout: lane l of the warp owns experts e = l + 32 c, c = 0..V-1 (coalesced loads of
// the row).  A selection takes K rounds; each round reduces every lane's best remaining
// (key, id) across the warp with XOR shuffles 16, 8, 4, 2, 1 under the total order (key
// desc, id asc), so every lane ends with the same winner, which its owner drops.  Lane k
// keeps slot k.
//
// Exact values only where they decide something.  Keys are first screened in cheap FP32
// (a fast sigmoid; logits that may carry an accumulation error `eps_l`), the K-th
// screened key fixes a window, and only the experts inside it -- the K selected ones and
// any close competitor -- get exact values: the logit re-evaluated by an error-free dot
// product when it was approximate (`refine`), and the correctly rounded sigmoid
// (evaluated in FP64 on those few lanes).  An expert outside the window is below every
// selected one even after the screening errors, so the final selection over the mixed
// keys equals the selection over exact keys, and the weights use exact values only.
#pragma once
#include "moe_internal.cuh"

namespace moe {

// Correctly rounded FP32 sigmoid from an FP64 evaluation (a disagreement with the
// correctly rounded value needs an FP64 error crossing an FP32 midpoint).  Out of line:
// it runs on a few lanes per row, and inlining FP64 exp everywhere bloats the routing
// kernels past the instruction cache.
__device__ __noinline__ float sigmoid_f32_rn(float l) { return __double2float_rn(1.0 / (1.0 + exp(-(double)l))); }
__device__ __noinline__ double exp_f64(double v) { return exp(v); }
// Screening sigmoid: a few ulp from the correctly rounded value.
__device__ __forceinline__ float sigmoid_fast(float l) { return __frcp_rn(1.0f + __expf(-l)); }

__device__ __forceinline__ bool key_better(float ka, int ia, float kb, int ib) {
    return ka > kb || (ka == kb && ia < ib);
}

// ---------------------------------------------------------------- error-free dot product
// Sum2 of Ogita, Rump and Oishi ("Accurate sum and dot product", SIAM J. Sci. Comput.
// 26(6), 2005): each BF16 x BF16 product is exact in FP32 (8-bit significands); the
// running sum takes it with Knuth's TwoSum, whose rounding error is exact and collected
// in a second FP32 term.  The pair (s, c) carries the sum with about twice FP32's
// precision; s + c rounded once is the correctly rounded dot product except within
// ~1e-12 (relative) of an FP32 rounding midpoint.
__device__ __forceinline__ void two_sum(float a, float b, float& s, float& e) {
    s = __fadd_rn(a, b);
    const float bb = __fsub_rn(s, a);
    e = __fadd_rn(__fsub_rn(a, __fsub_rn(s, bb)), __fsub_rn(b, bb));
}
struct Sum2 {
    float s, c;
};
__device__ __forceinline__ void sum2_add(Sum2& a, float p) {
    float q;
    two_sum(a.s, p, a.s, q);
    a.c = __fadd_rn(a.c, q);
}
__device__ __forceinline__ void sum2_dot8(Sum2& a, const uint4& x, const uint4& w) {
    sum2_add(a, __fmul_rn(bf16lo(x.x), bf16lo(w.x)));
    sum2_add(a, __fmul_rn(bf16hi(x.x), bf16hi(w.x)));
    sum2_add(a, __fmul_rn(bf16lo(x.y), bf16lo(w.y)));
    sum2_add(a, __fmul_rn(bf16hi(x.y), bf16hi(w.y)));
    sum2_add(a, __fmul_rn(bf16lo(x.z), bf16lo(w.z)));
    sum2_add(a, __fmul_rn(bf16hi(x.z), bf16hi(w.z)));
    sum2_add(a, __fmul_rn(bf16lo(x.w), bf16lo(w.w)));
    sum2_add(a, __fmul_rn(bf16hi(x.w), bf16hi(w.w)));
}
// Combine the lanes' pairs with TwoSum; every lane ends with the same bits (TwoSum's
// error term is unique, and the remaining adds are commutative pairs).
__device__ __forceinline__ float sum2_warp_finish(Sum2 a) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float s2 = __shfl_xor_sync(0xffffffffu, a.s, o);
        const float c2 = __shfl_xor_sync(0xffffffffu, a.c, o);
        float q;
        two_sum(a.s, s2, a.s, q);
        a.c = __fadd_rn(__fadd_rn(a.c, c2), q);
    }
    return __fadd_rn(a.s, a.c);
}
// Warp-collective correctly rounded dot product of two BF16 rows of length H (H % 8 == 0).
__device__ __noinline__ float warp_dot_exact(const bf16* __restrict__ a, const bf16* __restrict__ b, int H,
                                                int lane) {
    const int nch = H >> 3;
    Sum2 acc0 = {0.f, 0.f}, acc1 = {0.f, 0.f};
    int q = lane;
    for (; q + 32 < nch; q += 64) {
        const uint4 a0 = ld_nc16(a + (size_t)q * 8), b0 = ld_nc16(b + (size_t)q * 8);
        const uint4 a1 = ld_nc16(a + (size_t)(q + 32) * 8), b1 = ld_nc16(b + (size_t)(q + 32) * 8);
        sum2_dot8(acc0, a0, b0);
        sum2_dot8(acc1, a1, b1);
    }
    if (q < nch) sum2_dot8(acc0, ld_nc16(a + (size_t)q * 8), ld_nc16(b + (size_t)q * 8));
    float e;
    two_sum(acc0.s, acc1.s, acc0.s, e);
    acc0.c = __fadd_rn(__fadd_rn(acc0.c, acc1.c), e);
    return sum2_warp_finish(acc0);
}

// ---------------------------------------------------------------- selection
// Order-preserving map of an FP32 key to uint32 (larger key -> larger code; -0 and +0
// map to the same code so that they tie, as IEEE comparison has them).
__device__ __forceinline__ uint32_t key_code(float k) {
    uint32_t u = __float_as_uint(k);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// K rounds over the lane-strided keys.  Each round takes every lane's best remaining
// expert under (key desc, id asc) and reduces across the warp with two hardware
// reductions: the maximum key code, then the minimum id among the lanes holding it.
// Returns the id of slot `lane` (lanes < K) and the K-th key in every lane.
template <int V>
__device__ __forceinline__ int warp_select(const float (&key)[V], int E, int K, int lane, float& kth) {
    uint32_t avail = 0;
#pragma unroll
    for (int c = 0; c < V; ++c)
        if (lane + 32 * c < E) avail |= 1u << c;
    int my = 0;
    kth = 0.0f;
    for (int k = 0; k < K; ++k) {
        float bk = __int_as_float(0xff800000);
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
        const uint32_t code = (bi == 0x7fffffff) ? 0u : key_code(bk);
        const uint32_t best = __reduce_max_sync(0xffffffffu, code);
        const int win = (int)__reduce_min_sync(0xffffffffu, (code == best) ? (uint32_t)bi : 0x7fffffffu);
        if (lane == (win & 31)) avail &= ~(1u << (win >> 5));
        if (lane == k) my = win;
        if (k == K - 1) kth = __shfl_sync(0xffffffffu, bk, win & 31);
    }
    return my;
}

// Value of expert `id` (uniform across the warp) from its owner lane.
template <int V>
__device__ __forceinline__ float warp_fetch(const float (&v)[V], int id) {
    const int cw = id >> 5;
    float r = v[0];
#pragma unroll
    for (int c = 1; c < V; ++c)
        if (c == cw) r = v[c];
    return __shfl_sync(0xffffffffu, r, id & 31);
}

// Position of the n-th (0-based) set bit of m; n < popc(m).
__device__ __forceinline__ int nth_set_bit(unsigned m, int n) {
    int p = 0;
#pragma unroll
    for (int w = 16; w >= 1; w >>= 1) {
        const int lo = __popc(m & ((1u << w) - 1u));
        if (n >= lo) {
            n -= lo;
            m >>= w;
            p += w;
        }
    }
    return p;
}

struct NoRefine {
    __device__ float operator()(int) const { return 0.0f; }
};

// Screening + exact values for the candidates.  On entry key[] holds the screening keys;
// on exit the keys of every candidate are exact (and refined logits are in l).
template <int V, class Refine>
__device__ __forceinline__ void route_refine_keys(float (&l)[V], float (&key)[V], int E, int K, bool sig,
                                                  const float* bias, int lane, float eps_l, const Refine& refine) {
    const float NEG_INF = __int_as_float(0xff800000);
    float kth;
    warp_select<V>(key, E, K, lane, kth);
    // Window: screening error of a key (logit error, sigmoid slope <= 1/4, fast-sigmoid
    // error, key rounding), doubled because both sides of a comparison carry it.
    const float mag = fmaxf(1.0f, fabsf(kth));
    const float win = 2.0f * (sig ? (0.25f * eps_l + 4e-6f * mag) : (eps_l + 4e-7f * mag));
    const float lo = kth - win;
    unsigned mc[V];  // candidate lanes of each chunk
    int base[V];     // candidates in the chunks before
    int ncand = 0;
#pragma unroll
    for (int c = 0; c < V; ++c) {
        const int e = lane + 32 * c;
        const bool cand = e < E && !(key[c] < lo);
        mc[c] = __ballot_sync(0xffffffffu, cand);
        base[c] = ncand;
        ncand += __popc(mc[c]);
        if (eps_l > 0.0f) {
            unsigned m = mc[c];
            while (m) {
                const int src = __ffs(m) - 1;
                m &= m - 1;
                const float ex = refine(src + 32 * c);
                if (lane == src) l[c] = ex;
            }
        }
        if (!sig && cand) {
            float k = l[c];
            if (bias) k = __fadd_rn(k, bias[e]);
            key[c] = (k != k) ? NEG_INF : k;
        }
    }
    if (!sig) return;
    // Sigmoid keys: the candidates are packed onto consecutive lanes so that the FP64
    // sigmoid runs once per 32 candidates rather than once per chunk holding one.
    const unsigned lt = (1u << lane) - 1u;
    for (int r0 = 0; r0 < ncand; r0 += 32) {
        const int j = r0 + lane;  // candidate evaluated by this lane
        float lv = 0.0f;
#pragma unroll
        for (int c = 0; c < V; ++c) {
            const int rel = j - base[c];
            const bool mine = rel >= 0 && rel < __popc(mc[c]);
            const float v = __shfl_sync(0xffffffffu, l[c], mine ? nth_set_bit(mc[c], rel) : 0);
            if (mine) lv = v;
        }
        const float sv = (j < ncand) ? sigmoid_f32_rn(lv) : 0.0f;
#pragma unroll
        for (int c = 0; c < V; ++c) {
            const int pos = base[c] + __popc(mc[c] & lt) - r0;  // this lane's candidate, this round
            const bool here = ((mc[c] >> lane) & 1u) && pos >= 0 && pos < 32;
            const float got = __shfl_sync(0xffffffffu, sv, here ? pos : 0);
            if (here) {
                float k = got;
                if (bias) k = __fadd_rn(k, bias[lane + 32 * c]);
                key[c] = (k != k) ? NEG_INF : k;
            }
        }
    }
}

// Weights of the selected experts from exact values (lanes k < K hold slot k).
template <int V>
__device__ __forceinline__ void finish_route_row(const float (&l)[V], int E, int K, bool sig, int renorm, int lane,
                                                 int out_id, float& out_w, float& out_l) {
    const float NEG_INF = __int_as_float(0xff800000);
    out_l = 0.0f;
    for (int k = 0; k < K; ++k) {
        const int id = __shfl_sync(0xffffffffu, out_id, k);
        const float v = warp_fetch<V>(l, id);
        if (lane == k) out_l = v;
    }
    if (sig) {
        const float s = (lane < K) ? sigmoid_f32_rn(out_l) : 0.0f;
        double sum = 0.0;
        for (int k = 0; k < K; ++k) sum += (double)__shfl_sync(0xffffffffu, s, k);
        out_w = renorm ? __double2float_rn((double)s / sum) : s;
    } else {
        float lmax = NEG_INF;
#pragma unroll
        for (int c = 0; c < V; ++c)
            if (lane + 32 * c < E && l[c] == l[c]) lmax = fmaxf(lmax, l[c]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
        const double ex = (lane < K) ? exp_f64((double)out_l - (double)lmax) : 0.0;
        double sum = 0.0;
        if (renorm) {
            for (int k = 0; k < K; ++k) sum += __shfl_sync(0xffffffffu, ex, k);
        } else {  // full softmax: the other experts' terms in FP32 (not a workload mode)
            float part = 0.0f;
#pragma unroll
            for (int c = 0; c < V; ++c)
                if (lane + 32 * c < E) part += __expf(l[c] - lmax);
            part = warp_sum(part);
            sum = (double)part;
        }
        out_w = __double2float_rn(ex / sum);
    }
}

// One routing row.  l[c]: logit of expert lane + 32c (any value for e >= E), exact when
// eps_l == 0, otherwise within eps_l (absolute) of the exact FP32 value and re-evaluated
// with refine(e) (warp-collective) where it matters; refined logits are written back
// into l.  Outputs on lanes k < K: slot k's expert id, weight and exact logit.
template <int V, class Refine>
__device__ __forceinline__ void warp_route_row(float (&l)[V], int E, int K, int score, const float* bias, int renorm,
                                               int lane, float eps_l, const Refine& refine, int& out_id, float& out_w,
                                               float& out_l) {
    const float NEG_INF = __int_as_float(0xff800000);
    const bool sig = score == MOE_SCORE_SIGMOID;
    float key[V];
#pragma unroll
    for (int c = 0; c < V; ++c) {
        const int e = lane + 32 * c;
        key[c] = NEG_INF;
        if (e < E) {
            const float lv = l[c];
            float k = sig ? sigmoid_fast(lv) : lv;
            if (bias) k = __fadd_rn(k, bias[e]);
            key[c] = (k != k) ? NEG_INF : k;
        }
    }
    float kth;
    if (!sig && eps_l == 0.0f) {  // exact logits keyed directly: the screening keys are the keys
        out_id = warp_select<V>(key, E, K, lane, kth);
    } else {
        route_refine_keys<V>(l, key, E, K, sig, bias, lane, eps_l, refine);
        out_id = warp_select<V>(key, E, K, lane, kth);
    }
    finish_route_row<V>(l, E, K, sig, renorm, lane, out_id, out_w, out_l);
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

// V = ceil(E / 32) rounded up to a power of two (1..32).
__host__ __device__ inline int topk_v(int E) {
    int v = (E + 31) / 32;
    int p = 1;
    while (p < v) p <<= 1;
    return p;
}

}  // namespace moe
