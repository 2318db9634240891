// router.cu -- router logits for few tokens, the warp-per-row router top-k (moe_router_topk
// and the many-token path), and the route table of the few-token path.
#include "kernels.cuh"
#include "router.cuh"

namespace moe {

// Error bound of the tensor-core router logits of one token row.  The MMA forms every
// BF16 x BF16 product exactly in FP32 and accumulates a logit's H products (zero padding
// included) sixteen at a time: each tcgen05.mma of K = 16 adds its 16 products to the
// FP32 accumulator.  Model: one such step aligns its 17 addends to the largest and keeps
// at least 24 significant bits of it, truncating the rest, then rounds or truncates the
// sum to FP32 -- an error below 17 units of the largest addend plus one unit of the
// result, i.e. below 18 * 2^-23 * (|C| + sum |p|) for accumulator C.  Over the H / 16
// steps (each |C| <= sum_h |x_h w_h| =: S) the logit lies within 18 * 2^-23 * (H/16 + 1) * S
// = 1.125 * 2^-23 * (H + 16) * S of the exact sum; 1.25 is taken for margin.  Cauchy-
// Schwarz bounds S by |x_t|_2 * max_e |Wr[e]|_2; the prep kernel supplies upper bounds
// of max_e |Wr[e]|_2^2 and of every |x_t|_2^2 (FP32 sums of squares scaled up by
// (1 + 2^-8) to cover their own rounding, H <= 2^16).  A final factor (1 + 2^-8) covers the
// roundings of this product.  Each re-evaluated logit is checked against the bound.
__device__ __forceinline__ float tc_logit_bound(float xnorm2, int H, float wnorm2) {
    const float hpad = (float)(((H + 63) / 64) * 64);
    return 1.25f * (hpad + 16.0f) * 0x1p-23f * sqrtf(xnorm2) * sqrtf(wnorm2) * (1.0f + 0x1p-8f);
}

// Exact re-evaluation of one candidate's logit (warp-collective), written back into the
// logits buffer.  A re-evaluated logit that lies farther than the row's bound `eps` from
// its tensor-core value (`screen`) means the bound's hardware model does not hold; that
// sets MOE_DEVERR_ROUTER_BOUND (the routing of the call is then not guaranteed exact).
struct RowRefine {
    const bf16* xr;
    const bf16* wr;
    int H, E, row, lane;
    float* logits_rw;
    float eps;
    int* err;
    __device__ float operator()(int e, float screen) const {
        const float v = warp_dot_exact(xr, wr + (size_t)e * H, H, lane);
        if (lane == 0) {
            if (logits_rw) logits_rw[(size_t)row * E + e] = v;
            if (!(fabsf(v - screen) <= eps)) set_dev_error(err, MOE_DEVERR_ROUTER_BOUND);
        }
        return v;
    }
};

// Shared-expert gate of one token row (warp-collective): the exact logit x[row] . w
// (FP64 sum of the exact products, rounded once) through the correctly rounded sigmoid.
__device__ __forceinline__ void shared_gate_row(const GateArgs& g, int row, int lane) {
    const float l = warp_dot_exact(g.x + (size_t)row * g.H, g.w, g.H, lane);
    if (lane == 0) g.out[row] = sigmoid_f32_rn(l);
}

// ---------------------------------------------------------------- call prep
// First kernel of a many-token call.  CTA 0 zeroes the call's counters.  Before the
// tensor-core router (wr given), the grid's warps also take the E router rows and the T
// token rows of x, four rows per warp at a time: the FP32 sum of the H squares lies within a relative
// H * 2^-24 of the exact value and is scaled up by (1 + 2^-8) (H <= 2^16), so it is an
// upper bound.  Each CTA's maximum over router rows goes to wpart[blockIdx.x] (consumers
// take the maximum over the grid's entries: no atomics, nothing to zero first); a token
// row's bound goes to xn2[t].
__global__ void __launch_bounds__(256, 1) prep_kernel(int* __restrict__ counters, int n, int* __restrict__ counters2,
                                                   int n2, const bf16* __restrict__ wr, int E, int H,
                                                   float* __restrict__ wpart, const bf16* __restrict__ x, int T,
                                                   float* __restrict__ xn2) {
    // The router GEMM that follows reads nothing written here and waits for this kernel
    // only at its end: let it start now and run alongside.
    pdl_trigger();
    const int tid = threadIdx.x, lane = tid & 31;
    if (blockIdx.x == 0) {
        for (int i = tid; i < n; i += blockDim.x) counters[i] = 0;
        for (int i = tid; i < n2; i += blockDim.x) counters2[i] = 0;
    }
    if (wr) {
        __shared__ float s_max[8];
        float m = 0.0f;
        const int nw = (gridDim.x * blockDim.x) >> 5;
        // Four rows per pass, so that a lane keeps the loads of four rows in flight.
        constexpr int kRows = 4;
        for (int r0 = ((blockIdx.x * blockDim.x + tid) >> 5) * kRows; r0 < E + T; r0 += nw * kRows) {
            float ss[kRows];
#pragma unroll
            for (int j = 0; j < kRows; ++j) ss[j] = 0.0f;
            for (int c = lane; c < (H >> 3); c += 32) {
                uint4 v[kRows];
#pragma unroll
                for (int j = 0; j < kRows; ++j) {
                    const int r = r0 + j;
                    const bf16* row = r < E ? wr + (size_t)r * H : x + (size_t)(r - E) * H;
                    v[j] = r < E + T ? ld_nc16(row + (size_t)c * 8) : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int j = 0; j < kRows; ++j) ss[j] = dot8(v[j], v[j], ss[j]);
            }
#pragma unroll
            for (int j = 0; j < kRows; ++j) {
                const int r = r0 + j;
                const float b = warp_sum(ss[j]) * (1.0f + 0x1p-8f);
                if (r < E) m = fmaxf(m, b);
                else if (r < E + T && lane == 0) xn2[r - E] = b;
            }
        }
        if (lane == 0) s_max[tid >> 5] = m;
        __syncthreads();
        if (tid == 0) {
            for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, s_max[w]);
            wpart[blockIdx.x] = m;
        }
    }
}

int prep_grid(int E, int T, int num_sms) { return std::max(1, std::min(num_sms, cdiv(E + T, 32))); }

cudaError_t launch_prep(int* counters, int n, int* counters2, int n2, const bf16* wr, int E, int H, float* wpart,
                        const bf16* x, int T, float* xn2, int num_sms, cudaStream_t s) {
    return launch_k(prep_kernel, dim3(prep_grid(E, wr ? T : 0, num_sms)), dim3(256), 0, s, false, counters, n,
                    counters2, n2, wr, E, H, wpart, x, T, xn2);
}

// Upper bound of max_e |Wr[e]|_2^2 from the prep kernel's per-CTA maxima (warp-collective).
__device__ __forceinline__ float wnorm2_max(const float* __restrict__ wpart, int n, int lane) {
    float m = 0.0f;
    for (int i = lane; i < n; i += 32) m = fmaxf(m, wpart[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    return m;
}

// ---------------------------------------------------------------- top-k, one warp per row
static constexpr int kTopkRowsPerBlock = 4;  // small blocks: the SM fills up to its register limit

template <int V, bool BF16_IN, bool REFINE>
__global__ void __launch_bounds__(32 * kTopkRowsPerBlock) topk_kernel(const void* __restrict__ logits, int M, int E, int K, int score,
                                                   const float* __restrict__ bias, int renorm,
                                                   float* __restrict__ topk_w, int32_t* __restrict__ topk_ids,
                                                   int32_t* __restrict__ src_idx, float* __restrict__ w_copy,
                                                   int32_t* __restrict__ id_copy, const bf16* __restrict__ x,
                                                   const bf16* __restrict__ wr, int H, float* logits_rw,
                                                   const float* __restrict__ wpart, int nwpart,
                                                   const float* __restrict__ xn2, int* err,
                                                   int* __restrict__ counts, const GateArgs gate) {
    __shared__ float s_wbuf[kTopkRowsPerBlock][32];
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    float* wbuf = s_wbuf[threadIdx.x >> 5];
    if (row < M) {
        float l[V];
        if (BF16_IN)
            load_row_bf16<V>(static_cast<const uint16_t*>(logits) + (size_t)row * E, E, lane, l);
        else
            load_row_f32<V>(static_cast<const float*>(logits) + (size_t)row * E, E, lane, l);
        int id;
        float w, lg;
        if (REFINE) {
            const bf16* xr = x + (size_t)row * H;
            const float eps = tc_logit_bound(xn2[row], H, wnorm2_max(wpart, nwpart, lane));
            const RowRefine rf{xr, wr, H, E, row, lane, logits_rw, eps, err};
            warp_route_row<V>(l, E, K, score, bias, renorm, lane, eps, rf, wbuf, id, w, lg);
        } else {
            warp_route_row<V>(l, E, K, score, bias, renorm, lane, 0.0f, NoRefine{}, wbuf, id, w, lg);
        }
        if (lane < K) {
            const size_t o = (size_t)row * K + lane;
            topk_w[o] = w;
            topk_ids[o] = id;
            if (src_idx) src_idx[o] = lane * M + row;
            if (w_copy) w_copy[o] = w;
            if (id_copy) id_copy[o] = id;
            if (counts) atomicAdd(counts + id, 1);
        }
        if (gate.w) shared_gate_row(gate, row, lane);
    }
    pdl_trigger();
}

// ---------------------------------------------------------------- top-k, several warps per row
// For many experts and exact logits (few-token router, given or BF16 logits), one warp per
// row walks a long chain (V keys per lane, K rounds, rescans).  Here W warps share a row:
// warp w takes experts [w * Ew, (w + 1) * Ew) and selects their top K with the same
// screening and exact keys as a whole-row warp.  Every member of the row's top K is in its
// own warp's top K, so warp 0 then selects the row's top K from the W * K entries -- two per
// lane, compared by (exact key desc, expert id asc) with explicit ids -- and computes the
// weights (sigmoid: s_k / sum s; softmax with renorm: exp(l_k - l_max) / sum over the K).
static constexpr int kWideWarps = 4;
static constexpr int kWideMaxK = 16;  // W * K entries fit two per lane
template <int V, bool BF16_IN>
__global__ void __launch_bounds__(32 * kWideWarps) topk_wide_kernel(const void* __restrict__ logits, int M, int E,
                                                                    int K, int score, const float* __restrict__ bias,
                                                                    int renorm, float* __restrict__ topk_w,
                                                                    int32_t* __restrict__ topk_ids,
                                                                    int32_t* __restrict__ src_idx,
                                                                    float* __restrict__ w_copy,
                                                                    int32_t* __restrict__ id_copy,
                                                                    int* __restrict__ counts, const GateArgs gate) {
    __shared__ float s_wbuf[kWideWarps][32];
    __shared__ int s_id[kWideWarps][32];
    __shared__ float s_l[kWideWarps][32], s_s[kWideWarps][32];
    __shared__ int s_k[kWideWarps];
    pdl_wait();
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int row = blockIdx.x;
    const bool sig = score == MOE_SCORE_SIGMOID;
    const int ew = cdiv(cdiv(E, kWideWarps), 32) * 32;  // experts per warp (whole lanes)
    const int e0 = w * ew;
    const int en = max(0, min(ew, E - e0));
    const int kw = min(K, en);
    if (en > 0) {
        float l[V], key[V], sx[V];
        if (BF16_IN)
            load_row_bf16<V>(static_cast<const uint16_t*>(logits) + (size_t)row * E + e0, en, lane, l);
        else
            load_row_f32<V>(static_cast<const float*>(logits) + (size_t)row * E + e0, en, lane, l);
        const float* bw = bias ? bias + e0 : nullptr;
        screening_keys<V>(l, key, en, sig, bw, lane);
#pragma unroll
        for (int c = 0; c < V; ++c) sx[c] = 0.0f;
        if (sig) route_refine_keys<V>(l, key, sx, en, kw, sig, bw, lane, 0.0f, NoRefine{}, s_wbuf[w]);
        float kth, sel_l, sel_s;
        const int id = warp_select<V, true>(key, l, sx, en, kw, lane, kth, sel_l, sel_s);
        if (lane < kw) {
            s_id[w][lane] = e0 + id;
            s_l[w][lane] = sel_l;
            s_s[w][lane] = sel_s;
        }
    }
    if (lane == 0) s_k[w] = kw;
    __syncthreads();
    if (w == 1 && gate.w) shared_gate_row(gate, row, lane);  // alongside warp 0's merge
    if (w != 0) {
        pdl_trigger();
        return;
    }
    // ---- warp 0: the row's top K from the warps' entries, two per lane
    const float NEG_INF = __int_as_float(0xff800000);
    uint32_t code[2];
    int eid[2];
    float el[2], es[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int j = lane + 32 * h;  // entry j: warp j / K, slot j % K
        const int ww = j / K, kk = j - ww * K;
        code[h] = 0u;
        eid[h] = 0x7fffffff;
        el[h] = es[h] = 0.0f;
        if (ww < kWideWarps && kk < s_k[ww]) {
            eid[h] = s_id[ww][kk];
            el[h] = s_l[ww][kk];
            es[h] = s_s[ww][kk];
            float k = sig ? es[h] : el[h];
            if (bias) k = __fadd_rn(k, bias[eid[h]]);
            code[h] = key_code((k != k) ? NEG_INF : k);
        }
    }
    int my_id = 0;
    float my_l = 0.0f, my_s = 0.0f;
    for (int r = 0; r < K; ++r) {
        // this lane's better entry under (code desc, id asc); code 0 = none
        const bool second = code[1] > code[0] || (code[1] == code[0] && code[1] != 0u && eid[1] < eid[0]);
        const uint32_t c = second ? code[1] : code[0];
        const int id = second ? eid[1] : eid[0];
        const uint32_t best = __reduce_max_sync(0xffffffffu, c);
        const uint32_t mine = (c != 0u && c == best) ? (uint32_t)id : 0x7fffffffu;
        const int win = (int)__reduce_min_sync(0xffffffffu, mine);
        const int src = __ffs(__ballot_sync(0xffffffffu, c != 0u && c == best && id == win)) - 1;
        const float wl = __shfl_sync(0xffffffffu, second ? el[1] : el[0], src & 31);
        const float ws = __shfl_sync(0xffffffffu, second ? es[1] : es[0], src & 31);
        if (lane == r) {
            my_id = win;
            my_l = wl;
            my_s = ws;
        }
        if (lane == src) {
            if (second) code[1] = 0u;
            else code[0] = 0u;
        }
    }
    float wgt;
    if (sig) {
        const float sk = (lane < K) ? my_s : 0.0f;
        double sum = 0.0;
        for (int r = 0; r < K; ++r) sum += (double)__shfl_sync(0xffffffffu, sk, r);
        wgt = renorm ? __double2float_rn((double)sk / sum) : sk;
    } else {  // softmax with renorm (the only softmax mode routed here)
        float lmax = (lane < K) ? my_l : NEG_INF;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
        const double ex = (lane < K) ? exp_f64((double)my_l - (double)lmax) : 0.0;
        double sum = 0.0;
        for (int r = 0; r < K; ++r) sum += __shfl_sync(0xffffffffu, ex, r);
        wgt = __double2float_rn(ex / sum);
    }
    if (lane < K) {
        const size_t o = (size_t)row * K + lane;
        topk_w[o] = wgt;
        topk_ids[o] = my_id;
        if (src_idx) src_idx[o] = lane * M + row;
        if (w_copy) w_copy[o] = wgt;
        if (id_copy) id_copy[o] = my_id;
        if (counts) atomicAdd(counts + my_id, 1);
    }
    pdl_trigger();
}

// The several-warp top-k serves exact logits with many experts (at least 8 keys per lane
// in the one-warp form) when the weights need only the selected experts.
static bool use_wide_topk(int E, int K, int score, int renorm) {
    return E > 256 && K <= kWideMaxK && (score == MOE_SCORE_SIGMOID || renorm);
}

cudaError_t launch_topk(const void* logits, bool bf16_in, int M, int E, int K, int score, const float* bias,
                        int renorm, float* topk_w, int32_t* topk_ids, int32_t* src_idx, float* w_copy,
                        int32_t* id_copy, cudaStream_t s, bool pdl, const RefineArgs* refine, int* counts,
                        const GateArgs* gate_in) {
    dim3 grid(cdiv(M, kTopkRowsPerBlock)), block(32 * kTopkRowsPerBlock);
    const GateArgs gate = gate_in ? *gate_in : GateArgs{nullptr, nullptr, 0, nullptr};
    if (!refine && use_wide_topk(E, K, score, renorm)) {
        const int vw = topk_v(cdiv(E, kWideWarps));
#define MOE_W(VV)                                                                                                   \
        if (vw == VV)                                                                                               \
            return bf16_in ? launch_k(topk_wide_kernel<VV, true>, dim3(M), dim3(32 * kWideWarps), 0, s, pdl, logits, \
                                      M, E, K, score, bias, renorm, topk_w, topk_ids, src_idx, w_copy, id_copy,      \
                                      counts, gate)                                                                 \
                           : launch_k(topk_wide_kernel<VV, false>, dim3(M), dim3(32 * kWideWarps), 0, s, pdl, logits,\
                                      M, E, K, score, bias, renorm, topk_w, topk_ids, src_idx, w_copy, id_copy,      \
                                      counts, gate);
        MOE_W(4) MOE_W(8)
#undef MOE_W
    }
    const int v = topk_v(E);
    const bf16* x = refine ? refine->x : nullptr;
    const bf16* wr = refine ? refine->wr : nullptr;
    const int H = refine ? refine->H : 0;
    float* lrw = refine ? refine->logits_rw : nullptr;
    const float* wn2 = refine ? refine->wpart : nullptr;
    const int nwp = refine ? refine->nwpart : 0;
    const float* xn2 = refine ? refine->xn2 : nullptr;
    int* err = refine ? refine->err : nullptr;
#define MOE_L(VV)                                                                                              \
    if (v == VV) {                                                                                             \
        if (refine)                                                                                            \
            return launch_k(topk_kernel<VV, false, true>, grid, block, 0, s, pdl, logits, M, E, K, score, bias, \
                            renorm, topk_w, topk_ids, src_idx, w_copy, id_copy, x, wr, H, lrw, wn2, nwp, xn2,  \
                            err, counts, gate);                                                                \
        return bf16_in ? launch_k(topk_kernel<VV, true, false>, grid, block, 0, s, pdl, logits, M, E, K, score, \
                                  bias, renorm, topk_w, topk_ids, src_idx, w_copy, id_copy, x, wr, H, lrw, wn2, \
                                  nwp, xn2, err, counts, gate)                                                           \
                       : launch_k(topk_kernel<VV, false, false>, grid, block, 0, s, pdl, logits, M, E, K, score, \
                                  bias, renorm, topk_w, topk_ids, src_idx, w_copy, id_copy, x, wr, H, lrw, wn2, \
                                  nwp, xn2, err, counts, gate);                                                          \
    }
    MOE_L(1) MOE_L(2) MOE_L(4) MOE_L(8) MOE_L(16) MOE_L(32)
#undef MOE_L
    return cudaErrorInvalidValue;
}

// ---------------------------------------------------------------- top-k after the tensor-core router
// In three kernels, so that the exact re-evaluation of the candidates runs with one warp
// per candidate (thousands of independent dot products) instead of one warp walking its
// row's candidates one after another:
//   screen: warp per row; screening select on the tensor-core logits, and the row's
//           candidates (keys within the window of the K-th) appended to a global list
//           (one atomic per row reserves a contiguous range);
//   refine: warp per candidate; exact logit (FP64 sum of the exact products), written to
//           the list and back into the logits;
//   final:  warp per row; the candidates, one per lane, keyed on exact values (correctly
//           rounded sigmoid), top K by (key desc, id asc), weights, slot counts.
// The K selected are always candidates (see route_refine_keys), so the final select over
// the candidates alone is the select over exact keys.  A row with more than 32 candidates
// (not seen on any workload) is routed by the one-kernel path with per-row refinement.
template <int V>
__global__ void __launch_bounds__(32 * kTopkRowsPerBlock) topk_screen_kernel(const float* __restrict__ logits, int M,
                                                                              int E, int K, int score,
                                                                              const float* __restrict__ bias,
                                                                              const CandList cl,
                                                                              const bf16* __restrict__ x, int H,
                                                                              const float* __restrict__ wpart,
                                                                              int nwpart,
                                                                              const float* __restrict__ xn2) {
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (row < M) {
        const bool sig = score == MOE_SCORE_SIGMOID;
        float l[V], key[V];
        load_row_f32<V>(logits + (size_t)row * E, E, lane, l);
        const float eps = tc_logit_bound(xn2[row], H, wnorm2_max(wpart, nwpart, lane));
        if (lane == 0) cl.row_eps[row] = eps;
        screening_keys<V>(l, key, E, sig, bias, lane);
        float kth, ua, ub;
        warp_select<V, false>(key, key, key, E, K, lane, kth, ua, ub);
        const float lo = kth - screen_window(kth, sig, eps);
        unsigned mc[V];
        int before[V], n = 0;
#pragma unroll
        for (int c = 0; c < V; ++c) {
            mc[c] = __ballot_sync(0xffffffffu, lane + 32 * c < E && !(key[c] < lo));
            before[c] = n;
            n += __popc(mc[c]);
        }
        int base = 0;
        if (lane == 0) {
            base = atomicAdd(cl.count, n);
            cl.row_base[row] = base;
            cl.row_n[row] = n;
        }
        base = __shfl_sync(0xffffffffu, base, 0);
        const unsigned lt = (1u << lane) - 1u;
#pragma unroll
        for (int c = 0; c < V; ++c) {
            if ((mc[c] >> lane) & 1u) {
                const int pos = base + before[c] + __popc(mc[c] & lt);
                if (pos < cl.cap) {
                    cl.cand_row[pos] = row;
                    cl.cand_e[pos] = lane + 32 * c;
                }
            }
        }
    }
    pdl_trigger();
}

__global__ void __launch_bounds__(256) refine_kernel(const bf16* __restrict__ x, const bf16* __restrict__ wr, int M,
                                                    int H, int E, const CandList cl, float* __restrict__ logits_rw,
                                                    int* err) {
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int nw = (gridDim.x * blockDim.x) >> 5;
    const int n = min(*cl.count, cl.cap);
    for (int it = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; it < n; it += nw) {
        const int row = cl.cand_row[it], e = cl.cand_e[it];
        if ((unsigned)row >= (unsigned)M || (unsigned)e >= (unsigned)E) {
            if (lane == 0) set_dev_error(err, MOE_DEVERR_BAD_INDEX);
            continue;
        }
        const float v = warp_dot_exact(x + (size_t)row * H, wr + (size_t)e * H, H, lane);
        if (lane == 0) {
            cl.cand_val[it] = v;
            if (logits_rw) {  // the tensor-core value must lie within the row's bound
                const float screen = logits_rw[(size_t)row * E + e];
                if (!(fabsf(v - screen) <= cl.row_eps[row])) set_dev_error(err, MOE_DEVERR_ROUTER_BOUND);
                logits_rw[(size_t)row * E + e] = v;
            }
        }
    }
    pdl_trigger();
}

template <int V>
__global__ void __launch_bounds__(32 * kTopkRowsPerBlock) topk_final_kernel(
    const float* __restrict__ logits, int M, int E, int K, int score, const float* __restrict__ bias, int renorm,
    const CandList cl, float* __restrict__ topk_w, int32_t* __restrict__ topk_ids, float* __restrict__ w_copy,
    int32_t* __restrict__ id_copy, int* __restrict__ counts, const bf16* __restrict__ x,
    const bf16* __restrict__ wr, int H, float* logits_rw, int* err, const GateArgs gate) {
    __shared__ float s_wbuf[kTopkRowsPerBlock][32];
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (row >= M) {
        pdl_trigger();
        return;
    }
    const bool sig = score == MOE_SCORE_SIGMOID;
    const int n = cl.row_n[row], base = cl.row_base[row];
    int id = 0;
    float w = 0.0f;
    if (n <= 32 && base + n <= cl.cap) {
        const float NEG_INF = __int_as_float(0xff800000);
        const bool has = lane < n;
        const int e = has ? cl.cand_e[base + lane] : 0x7fffffff;
        const float lv = has ? cl.cand_val[base + lane] : 0.0f;
        const float sv = (has && sig) ? sigmoid_f32_rn(lv) : 0.0f;
        float k = sig ? sv : lv;
        if (has && bias) k = __fadd_rn(k, bias[e]);
        const uint32_t code0 = has ? key_code((k != k) ? NEG_INF : k) : 0u;
        uint32_t code = code0;
        float sel_l = 0.0f, sel_s = 0.0f;
        for (int r = 0; r < K; ++r) {  // K rounds over one candidate per lane
            const uint32_t best = __reduce_max_sync(0xffffffffu, code);
            const uint32_t mine = (code != 0u && code == best) ? (uint32_t)e : 0x7fffffffu;
            const int win = (int)__reduce_min_sync(0xffffffffu, mine);
            const int src = __ffs(__ballot_sync(0xffffffffu, code != 0u && e == win)) - 1;
            const float wl = __shfl_sync(0xffffffffu, lv, src & 31);
            const float ws = __shfl_sync(0xffffffffu, sv, src & 31);
            if (lane == r) {
                id = win;
                sel_l = wl;
                sel_s = ws;
            }
            if (lane == src) code = 0u;
        }
        if (sig) {
            const float sk = (lane < K) ? sel_s : 0.0f;
            double sum = 0.0;
            for (int r = 0; r < K; ++r) sum += (double)__shfl_sync(0xffffffffu, sk, r);
            w = renorm ? __double2float_rn((double)sk / sum) : sk;
        } else {  // softmax with renorm (the only softmax mode routed here)
            float lmax = (lane < K) ? sel_l : NEG_INF;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
            const double ex = (lane < K) ? exp_f64((double)sel_l - (double)lmax) : 0.0;
            double sum = 0.0;
            for (int r = 0; r < K; ++r) sum += __shfl_sync(0xffffffffu, ex, r);
            w = __double2float_rn(ex / sum);
        }
    } else {  // many candidates: route the row in one warp with per-candidate refinement
        float l[V];
        load_row_f32<V>(logits + (size_t)row * E, E, lane, l);
        const float eps = cl.row_eps[row];
        const RowRefine rf{x + (size_t)row * H, wr, H, E, row, lane, logits_rw, eps, err};
        float lg;
        warp_route_row<V>(l, E, K, score, bias, renorm, lane, eps, rf, s_wbuf[threadIdx.x >> 5], id, w, lg);
    }
    if (lane < K) {
        const size_t o = (size_t)row * K + lane;
        topk_w[o] = w;
        topk_ids[o] = id;
        if (w_copy) w_copy[o] = w;
        if (id_copy) id_copy[o] = id;
        if (counts) atomicAdd(counts + id, 1);
    }
    if (gate.w) shared_gate_row(gate, row, lane);
    pdl_trigger();
}

cudaError_t launch_topk_split(const float* logits, int M, int E, int K, int score, const float* bias, int renorm,
                              float* topk_w, int32_t* topk_ids, float* w_copy, int32_t* id_copy, const CandList& cl,
                              const RefineArgs& ra, int* counts, int* err, int num_sms, cudaStream_t s, bool pdl,
                              const std::function<bool()>* mark, const GateArgs& gate) {
    dim3 grid(cdiv(M, kTopkRowsPerBlock)), block(32 * kTopkRowsPerBlock);
    const int v = topk_v(E);
    cudaError_t st = cudaErrorInvalidValue;
#define MOE_S(VV)                                                                                           \
    if (v == VV)                                                                                            \
        st = launch_k(topk_screen_kernel<VV>, grid, block, 0, s, pdl, logits, M, E, K, score, bias, cl, ra.x, \
                      ra.H, ra.wpart, ra.nwpart, ra.xn2);
    MOE_S(1) MOE_S(2) MOE_S(4) MOE_S(8) MOE_S(16) MOE_S(32)
#undef MOE_S
    if (st != cudaSuccess) return st;
    if (mark && !(*mark)()) return cudaErrorUnknown;
    st = launch_k(refine_kernel, dim3(num_sms * 8), dim3(256), 0, s, pdl, ra.x, ra.wr, M, ra.H, E, cl,
                  ra.logits_rw, err);
    if (st != cudaSuccess) return st;
    if (mark && !(*mark)()) return cudaErrorUnknown;
    st = cudaErrorInvalidValue;
#define MOE_F(VV)                                                                                             \
    if (v == VV)                                                                                              \
        st = launch_k(topk_final_kernel<VV>, grid, block, 0, s, pdl, logits, M, E, K, score, bias, renorm, cl, \
                      topk_w, topk_ids, w_copy, id_copy, counts, ra.x, ra.wr, ra.H, ra.logits_rw, err, gate);
    MOE_F(1) MOE_F(2) MOE_F(4) MOE_F(8) MOE_F(16) MOE_F(32)
#undef MOE_F
    return st;
}

// ---------------------------------------------------------------- router logits, few tokens
// l[t, e] = x[t,:] . Wr[e,:]: each BF16 x BF16 product is exact in FP32 and is summed in
// FP64, rounded once to FP32 (the oracle's definition; see warp_dot_exact).  CTA (i, g):
// two warps, one expert row each (experts 2i, 2i+1) held in registers (one memory latency
// per row), and token group g of kRouterTokBlock tokens, staged in shared memory by one
// bulk copy.  Each warp runs four independent FP64 chains (two tokens x even/odd chunks).
// Splitting the tokens over the grid keeps the chains short: the arithmetic, not memory,
// would otherwise set the time at T = 16..64.
static constexpr int kRouterTokBlock = 4;

template <int VH>
__global__ void __launch_bounds__(64) router_logits_small(const bf16* __restrict__ x, const bf16* __restrict__ wr,
                                                          int T, int H, int E, float* __restrict__ logits,
                                                          float* __restrict__ logits_copy, int* err,
                                                          int* __restrict__ zero_ints, int n_zero,
                                                          int* __restrict__ zero_ints2, int n_zero2) {
    extern __shared__ uint4 xs[];  // [kRouterTokBlock][H / 8]
    __shared__ __align__(8) uint64_t s_bar;
    __shared__ int s_abort;
    const int tid = threadIdx.x, lane = tid & 31;
    // As the first kernel of a many-token call, CTA (0, 0) also zeroes the call's counters.
    if (zero_ints && blockIdx.x == 0 && blockIdx.y == 0) {
        for (int i = tid; i < n_zero; i += blockDim.x) zero_ints[i] = 0;
        for (int i = tid; i < n_zero2; i += blockDim.x) zero_ints2[i] = 0;
    }
    const uint32_t bar = smem_u32(&s_bar);
    if (tid == 0) {
        mbar_init(bar, 1);
        s_abort = 0;
        fence_mbar_init();
    }
    const int e = blockIdx.x * (blockDim.x >> 5) + (tid >> 5);
    const int nch = H >> 3;
    uint4 w[VH];
#pragma unroll
    for (int j = 0; j < VH; ++j) {
        const int c = lane + 32 * j;
        w[j] = (e < E && c < nch) ? ld_stream16(wr + (size_t)e * H + (size_t)c * 8) : make_uint4(0u, 0u, 0u, 0u);
    }
    pdl_wait();  // x may come from the previous kernel
    const int t0 = blockIdx.y * kRouterTokBlock;
    const int nt = min(kRouterTokBlock, T - t0);
    __syncthreads();  // the barrier init is visible
    if (tid == 0) {   // the token group in one bulk copy (rows are 16-byte multiples)
        const uint32_t bytes = (uint32_t)nt * H * 2;
        mbar_expect_tx(bar, bytes);
        bulk_copy_g2s(smem_u32(xs), x + (size_t)t0 * H, bytes, bar);
    }
    const bool ok = mbar_wait(bar, 0, &s_abort, err);
    if (ok && e < E) {
        for (int t = 0; t < nt; t += 2) {
            const bool two = t + 1 < nt;
            double a0 = 0.0, a1 = 0.0, b0 = 0.0, b1 = 0.0;
#pragma unroll
            for (int j = 0; j < VH; ++j) {
                const int c = lane + 32 * j;
                if (c < nch) {
                    const uint4 xa = xs[t * nch + c];
                    if (j & 1) a1 = dot8_f64p(xa, w[j], a1);
                    else a0 = dot8_f64p(xa, w[j], a0);
                    if (two) {
                        const uint4 xb = xs[(t + 1) * nch + c];
                        if (j & 1) b1 = dot8_f64p(xb, w[j], b1);
                        else b0 = dot8_f64p(xb, w[j], b0);
                    }
                }
            }
            const float va = __double2float_rn(warp_sum_f64(a0 + a1));
            const float vb = __double2float_rn(warp_sum_f64(b0 + b1));
            if (lane == 0) {
                logits[(size_t)(t0 + t) * E + e] = va;
                if (logits_copy) logits_copy[(size_t)(t0 + t) * E + e] = va;
                if (two) {
                    logits[(size_t)(t0 + t + 1) * E + e] = vb;
                    if (logits_copy) logits_copy[(size_t)(t0 + t + 1) * E + e] = vb;
                }
            }
        }
    }
    __syncthreads();
    if (s_abort) {  // a wait gave up: let the bulk copy in flight land before the CTA retires
        const uint64_t ts = globaltimer_ns();
        while (globaltimer_ns() - ts < 50000ull) {
        }
    }
    pdl_trigger();
}

bool router_small_supported(int H) { return (H >> 3) <= 32 * 16; }

cudaError_t launch_router_small(const bf16* x, const bf16* wr, int T, int H, int E, float* logits,
                                float* logits_copy, int* err, cudaStream_t s, bool pdl, int* zero_ints, int n_zero,
                                int* zero_ints2, int n_zero2) {
    dim3 grid(cdiv(E, 2), cdiv(T, kRouterTokBlock)), block(64);
    const size_t smem = (size_t)kRouterTokBlock * H * 2;
    const int need = cdiv(H >> 3, 32);
#define MOE_R(VV)                                                                                                \
    if (need <= VV) {                                                                                            \
        cudaError_t st = cudaFuncSetAttribute(router_logits_small<VV>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                                               (int)smem);                                                       \
        if (st != cudaSuccess) return st;                                                                        \
        return launch_k(router_logits_small<VV>, grid, block, smem, s, pdl, x, wr, T, H, E, logits, logits_copy, err, \
                        zero_ints, n_zero, zero_ints2, n_zero2);                                                 \
    }
    MOE_R(4) MOE_R(8) MOE_R(12) MOE_R(16)
#undef MOE_R
    return cudaErrorInvalidValue;
}

// ---------------------------------------------------------------- route table, few tokens
// One CTA, one warp per token row: route each row, then list the distinct experts in
// ascending order with the slots (k*T + t) each one serves, for the streaming kernels.
// Everything is built in shared memory and written out once.
template <int V>
__global__ void __launch_bounds__(32 * kSmallMaxT) route_small_kernel(const float* __restrict__ logits, int T, int E,
                                                                      int K, int score, const float* __restrict__ bias,
                                                                      int renorm, RouteTable* __restrict__ rt,
                                                                      float* __restrict__ w_out,
                                                                      int32_t* __restrict__ id_out,
                                                                      const GateArgs gate) {
    __shared__ int s_ids[kSmallMaxSlots];
    __shared__ int s_uidx[MOE_MAX_EXPERTS];
    __shared__ int s_ulist[kSmallMaxSlots];
    __shared__ int s_uoff[kSmallMaxSlots + 1];
    __shared__ int s_wcnt[32], s_wbase[32];
    __shared__ float s_wbuf[kSmallMaxT][32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const int TK = T * K;
    for (int e = tid; e < E; e += blockDim.x) s_uidx[e] = 0;
    pdl_wait();
    for (int t = warp; t < T; t += nw) {
        float l[V];
        load_row_f32<V>(logits + (size_t)t * E, E, lane, l);
        int id;
        float w, lg;
        warp_route_row<V>(l, E, K, score, bias, renorm, lane, 0.0f, NoRefine{}, s_wbuf[warp], id, w, lg);
        if (lane < K) {
            s_ids[t * K + lane] = id;
            rt->ids[t * K + lane] = id;
            rt->w[t * K + lane] = w;
            if (w_out) w_out[(size_t)t * K + lane] = w;
            if (id_out) id_out[(size_t)t * K + lane] = id;
        }
        if (gate.w) shared_gate_row(gate, t, lane);  // gate.out = rt->gate
    }
    __syncthreads();
    for (int i = tid; i < TK; i += blockDim.x) atomicAdd(&s_uidx[s_ids[i]], 1);  // slots per expert
    __syncthreads();
    const int nchunk = cdiv(E, 32);
    for (int j = warp; j < nchunk; j += nw) {
        const int e = 32 * j + lane;
        const unsigned m = __ballot_sync(0xffffffffu, e < E && s_uidx[e] > 0);
        if (lane == 0) s_wcnt[j] = __popc(m);
    }
    __syncthreads();
    if (warp == 0) {
        const int v = (lane < nchunk) ? s_wcnt[lane] : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += n;
        }
        if (lane < nchunk) s_wbase[lane] = incl - v;
    }
    __syncthreads();
    for (int j = warp; j < nchunk; j += nw) {  // compact the experts, ascending id
        const int e = 32 * j + lane;
        const bool f = e < E && s_uidx[e] > 0;
        const unsigned m = __ballot_sync(0xffffffffu, f);
        if (f) s_ulist[s_wbase[j] + __popc(m & ((1u << lane) - 1u))] = e;
    }
    __syncthreads();
    const int U = s_wbase[nchunk - 1] + s_wcnt[nchunk - 1];
    if (warp == 0) {  // offsets of each expert's slot list
        int run = 0;
        for (int u0 = 0; u0 < U; u0 += 32) {
            const int u = u0 + lane;
            const int v = (u < U) ? s_uidx[s_ulist[u]] : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += n;
            }
            if (u < U) s_uoff[u] = run + incl - v;
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) s_uoff[U] = run;
    }
    __syncthreads();
    for (int u = tid; u < U; u += blockDim.x) {  // one thread per expert: its slots, ascending token
        const int e = s_ulist[u];
        int pos = s_uoff[u];
        rt->ulist[u] = e;
        rt->uoff[u] = pos;
        for (int t = 0; t < T; ++t)
            for (int k = 0; k < K; ++k)
                if (s_ids[t * K + k] == e) rt->utok[pos++] = k * T + t;
    }
    if (tid == 0) {
        rt->uoff[U] = s_uoff[U];
        rt->U = U;
    }
    pdl_trigger();
}

cudaError_t launch_route_small(const float* logits, int T, int E, int K, int score, const float* bias, int renorm,
                               RouteTable* rt, float* w_out, int32_t* id_out, cudaStream_t s, bool pdl,
                               const GateArgs& gate) {
    const int v = topk_v(E);
    dim3 grid(1), block(32 * std::max(1, std::min(T, kSmallMaxT)));
#define MOE_RT(VV)                                                                                              \
    if (v == VV)                                                                                                \
        return launch_k(route_small_kernel<VV>, grid, block, 0, s, pdl, logits, T, E, K, score, bias, renorm, rt, \
                        w_out, id_out, gate);
    MOE_RT(1) MOE_RT(2) MOE_RT(4) MOE_RT(8) MOE_RT(16) MOE_RT(32)
#undef MOE_RT
    return cudaErrorInvalidValue;
}

}  // namespace moe
