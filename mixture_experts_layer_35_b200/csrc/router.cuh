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
// entry across the warp under the total order (key desc, id asc) -- the maximum
// order-preserving key code, then the minimum id among the lanes holding it, two
// hardware warp reductions -- so every lane sees the same winner, which its owner drops.
// Lane k keeps slot k.
//
// Exact values only where they decide something.  Keys are first screened in cheap FP32
// (a fast sigmoid; logits that may carry an accumulation error `eps_l`), the K-th
// screened key fixes a window, and only the experts inside it -- the K selected ones and
// any close competitor -- get exact values: the logit re-evaluated by an exact dot
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

// ---------------------------------------------------------------- exact dot product
// Warp-collective dot product of two BF16 rows of length H (H % 8 == 0), rounded once to
// FP32.  Each BF16 x BF16 product is exact in FP32 and is accumulated in FP64 (error about
// H * 2^-53 * sum|p|, far below half an FP32 ulp of the result except within that distance
// of a rounding midpoint, where the oracle's own FP64 sum has the same blind spot).  FP64
// runs at half the FP32 rate here, so one conversion and one add per product cost less
// than a compensated (TwoSum) FP32 accumulation, which measured slower.
__device__ __noinline__ float warp_dot_exact(const bf16* __restrict__ a, const bf16* __restrict__ b, int H,
                                                int lane) {
    const int nch = H >> 3;
    double acc0 = 0.0, acc1 = 0.0;
    int q = lane;
    for (; q + 32 < nch; q += 64) {
        const uint4 a0 = ld_nc16(a + (size_t)q * 8), b0 = ld_nc16(b + (size_t)q * 8);
        const uint4 a1 = ld_nc16(a + (size_t)(q + 32) * 8), b1 = ld_nc16(b + (size_t)(q + 32) * 8);
        acc0 = dot8_f64p(a0, b0, acc0);
        acc1 = dot8_f64p(a1, b1, acc1);
    }
    if (q < nch) acc0 = dot8_f64p(ld_nc16(a + (size_t)q * 8), ld_nc16(b + (size_t)q * 8), acc0);
    return __double2float_rn(warp_sum_f64(acc0 + acc1));
}

// ---------------------------------------------------------------- selection
// Order-preserving map of an FP32 key to uint32 (larger key -> larger code; -0 and +0
// map to the same code so that they tie, as IEEE comparison has them).
__device__ __forceinline__ uint32_t key_code(float k) {
    uint32_t u = __float_as_uint(k);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Inverse of key_code (zero decodes as +0).
__device__ __forceinline__ float key_decode(uint32_t code) {
    return __uint_as_float((code & 0x80000000u) ? (code & 0x7fffffffu) : ~code);
}

// One entry of a lane's selection cache: key code (0 = none: real keys never map to 0),
// chunk index, and two payload values that the selection hands to the slot's lane.
struct SelEntry {
    uint32_t code;
    int j;
    float pa, pb;
};

// K rounds over the lane-strided keys under (key desc, id asc).  Each lane keeps its
// three best remaining entries.  A round reduces the lanes' heads across the warp with
// two hardware reductions (the maximum code, then the minimum id among the lanes holding
// it); the winner's payload goes to lane k by shuffle.  The winning lane pops its head
// and rescans its keys only when its cache runs dry, so a round costs a few instructions
// instead of a scan of all V keys.
// Returns the id of slot `lane` (lanes < K), its payload (PAYLOAD), and the K-th key.
template <int V, bool PAYLOAD>
__device__ __forceinline__ int warp_select(const float (&key)[V], const float (&pa)[V], const float (&pb)[V], int E,
                                           int K, int lane, float& kth, float& out_a, float& out_b) {
    uint32_t avail = 0;
#pragma unroll
    for (int c = 0; c < V; ++c)
        if (lane + 32 * c < E) avail |= 1u << c;
    SelEntry e1, e2, e3;
    auto rescan = [&]() {
        e1 = e2 = e3 = SelEntry{0u, 0, 0.0f, 0.0f};
#pragma unroll
        for (int c = 0; c < V; ++c) {
            if ((avail >> c) & 1u) {
                // ids ascend with c within a lane: on equal codes the earlier entry ranks first
                const SelEntry n{key_code(key[c]), c, PAYLOAD ? pa[c] : 0.0f, PAYLOAD ? pb[c] : 0.0f};
                if (n.code > e1.code) {
                    e3 = e2;
                    e2 = e1;
                    e1 = n;
                } else if (n.code > e2.code) {
                    e3 = e2;
                    e2 = n;
                } else if (n.code > e3.code) {
                    e3 = n;
                }
            }
        }
    };
    rescan();
    int my = 0;
    out_a = out_b = 0.0f;
    kth = 0.0f;
    for (int k = 0; k < K; ++k) {
        const uint32_t best = __reduce_max_sync(0xffffffffu, e1.code);
        const uint32_t mine = (e1.code != 0u && e1.code == best) ? (uint32_t)(lane + 32 * e1.j) : 0x7fffffffu;
        const int win = (int)__reduce_min_sync(0xffffffffu, mine);
        if (PAYLOAD) {
            const float va = __shfl_sync(0xffffffffu, e1.pa, win & 31);
            const float vb = __shfl_sync(0xffffffffu, e1.pb, win & 31);
            if (lane == k) {
                out_a = va;
                out_b = vb;
            }
        }
        if (lane == k) my = win;
        if (k == K - 1) kth = key_decode(best);
        if (lane == (win & 31)) {
            avail &= ~(1u << (win >> 5));
            e1 = e2;
            e2 = e3;
            e3.code = 0u;
            if (e1.code == 0u && avail) rescan();
        }
    }
    return my;
}

// Window around the K-th screening key: the screening error of a key (logit error eps_l,
// sigmoid slope <= 1/4, fast-sigmoid error, key rounding), doubled because both sides of a
// comparison carry it.
__device__ __forceinline__ float screen_window(float kth, bool sig, float eps_l) {
    const float mag = fmaxf(1.0f, fabsf(kth));
    return 2.0f * (sig ? (0.25f * eps_l + 4e-6f * mag) : (eps_l + 4e-7f * mag));
}

// Screening keys of one row (fast sigmoid for sigmoid scores; -inf past E and for NaN).
template <int V>
__device__ __forceinline__ void screening_keys(const float (&l)[V], float (&key)[V], int E, bool sig,
                                               const float* bias, int lane) {
    const float NEG_INF = __int_as_float(0xff800000);
#pragma unroll
    for (int c = 0; c < V; ++c) {
        const int e = lane + 32 * c;
        key[c] = NEG_INF;
        if (e < E) {
            float k = sig ? sigmoid_fast(l[c]) : l[c];
            if (bias) k = __fadd_rn(k, bias[e]);
            key[c] = (k != k) ? NEG_INF : k;
        }
    }
}

struct NoRefine {
    __device__ float operator()(int, float) const { return 0.0f; }
};

// Screening + exact values for the candidates.  On entry key[] holds the screening keys;
// on exit the keys of every candidate are exact (and refined logits are in l), and for
// sigmoid scores sx[] holds each candidate's correctly rounded sigmoid.  The experts the
// final selection takes are always candidates: each of the K screened best has an exact
// key at least kth - win/2, above the exact key of anything outside the window.
// wbuf: 32 floats of shared memory owned by this warp.
template <int V, class Refine>
__device__ __forceinline__ void route_refine_keys(float (&l)[V], float (&key)[V], float (&sx)[V], int E, int K,
                                                  bool sig, const float* bias, int lane, float eps_l,
                                                  const Refine& refine, float* wbuf) {
    const float NEG_INF = __int_as_float(0xff800000);
    float kth, ua, ub;
    warp_select<V, false>(key, key, key, E, K, lane, kth, ua, ub);
    // Window: screening error of a key (logit error, sigmoid slope <= 1/4, fast-sigmoid
    // error, key rounding), doubled because both sides of a comparison carry it.
    const float lo = kth - screen_window(kth, sig, eps_l);
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
                const float screen = __shfl_sync(0xffffffffu, l[c], src);
                const float ex = refine(src + 32 * c, screen);
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
    // Sigmoid keys: the candidates' logits are packed into the warp's buffer, each lane
    // evaluates one FP64 sigmoid, and the results go back to the owners -- one pass per 32
    // candidates.
    const unsigned lt = (1u << lane) - 1u;
    for (int r0 = 0; r0 < ncand; r0 += 32) {
#pragma unroll
        for (int c = 0; c < V; ++c) {
            const int pos = base[c] + __popc(mc[c] & lt) - r0;
            if (((mc[c] >> lane) & 1u) && pos >= 0 && pos < 32) wbuf[pos] = l[c];
        }
        __syncwarp();
        const float lv = wbuf[lane];
        const float sv = (r0 + lane < ncand) ? sigmoid_f32_rn(lv) : 0.0f;
        __syncwarp();
        wbuf[lane] = sv;
        __syncwarp();
#pragma unroll
        for (int c = 0; c < V; ++c) {
            const int pos = base[c] + __popc(mc[c] & lt) - r0;
            if (((mc[c] >> lane) & 1u) && pos >= 0 && pos < 32) {
                const float sg = wbuf[pos];
                sx[c] = sg;
                float k = sg;
                if (bias) k = __fadd_rn(k, bias[lane + 32 * c]);
                key[c] = (k != k) ? NEG_INF : k;
            }
        }
        __syncwarp();
    }
}

// Weights of the selected experts from exact values: lane k < K holds slot k's logit
// sel_l and (sigmoid scores) its correctly rounded sigmoid sel_s.
template <int V>
__device__ __forceinline__ void finish_route_row(const float (&l)[V], int E, int K, bool sig, int renorm, int lane,
                                                 float sel_l, float sel_s, float& out_w) {
    const float NEG_INF = __int_as_float(0xff800000);
    if (sig) {
        const float s = (lane < K) ? sel_s : 0.0f;
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
        const double ex = (lane < K) ? exp_f64((double)sel_l - (double)lmax) : 0.0;
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
// with refine(e, screening value) (warp-collective) where it matters; refined logits are
// written back into l.  wbuf: 32 floats of shared memory owned by this warp.  Outputs on lanes k < K:
// slot k's expert id, weight and exact logit.
template <int V, class Refine>
__device__ __forceinline__ void warp_route_row(float (&l)[V], int E, int K, int score, const float* bias, int renorm,
                                               int lane, float eps_l, const Refine& refine, float* wbuf, int& out_id,
                                               float& out_w, float& out_l) {
    const float NEG_INF = __int_as_float(0xff800000);
    const bool sig = score == MOE_SCORE_SIGMOID;
    float key[V];
    float sx[V];  // exact sigmoid of the candidates (sigmoid scores only)
    screening_keys<V>(l, key, E, sig, bias, lane);
#pragma unroll
    for (int c = 0; c < V; ++c) sx[c] = 0.0f;
    // exact logits keyed directly (softmax, eps 0): the screening keys are the keys
    if (sig || eps_l > 0.0f) route_refine_keys<V>(l, key, sx, E, K, sig, bias, lane, eps_l, refine, wbuf);
    float kth, sel_s;
    out_id = warp_select<V, true>(key, l, sx, E, K, lane, kth, out_l, sel_s);
    finish_route_row<V>(l, E, K, sig, renorm, lane, out_l, sel_s, out_w);
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
