// stream.cu -- the few-token path: only the routed experts' weights are read, each
// exactly once from HBM, by 16-byte coalesced loads spread over every SM.  Dot products
// run on the CUDA cores with warp-level XOR reductions; there is no split-K reduce
// kernel (weight-streaming design of the vLLM PR #64636 skinny GEMM, "Overview", applied
// to the routed experts).
//
//   fc1_small: every CTA recomputes the routing of the T <= 16 tokens from the FP32
//              logits (cheap, deterministic, identical in every CTA), builds the sorted
//              list of distinct experts, and streams its share of the (expert, row)
//              items: h[slot, i] = act(W13[e] x)[i], plus the shared expert's rows.
//   fc2_small: each CTA owns a slice of output features f.  For every token it sums
//              w[t,k] * (W2[e_k, f, :] . h[slot]) in FP32 over the slots, rounds to BF16,
//              adds the BF16 shared-expert output and rounds again ("MTP1 isolated
//              gather/shared-add closure": routed FP32 accumulation -> BF16 -> shared BF16
//              add -> BF16), writing the layer output directly.  fc1 has already
//              prefetched the routed experts' W2 into L2 while it streamed W13.
#include "kernels.cuh"
#include "router.cuh"

namespace moe {

static constexpr int kSmallMaxSlots = kSmallMaxT * MOE_MAX_TOPK;

// Routing of all T tokens into shared memory: s_ids/s_w[t*K + k].
__device__ __forceinline__ void small_routing(const SmallArgs& a, int* s_ids, float* s_w, bool write_global) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    for (int t = warp; t < a.T; t += nw) {
        int id;
        float w, lg;
        warp_topk_f32(a.logits + (size_t)t * a.E, a.E, a.K, a.score, a.bias, a.renorm, lane, id, w, lg);
        if (lane < a.K) {
            s_ids[t * a.K + lane] = id;
            s_w[t * a.K + lane] = w;
            if (write_global) {
                if (a.w_out) a.w_out[(size_t)t * a.K + lane] = w;
                if (a.id_out) a.id_out[(size_t)t * a.K + lane] = id;
            }
        }
    }
}

template <int VH>
__global__ void __launch_bounds__(256) fc1_small(const SmallArgs a) {
    __shared__ int s_ids[kSmallMaxSlots];
    __shared__ float s_w[kSmallMaxSlots];
    __shared__ int s_uidx[MOE_MAX_EXPERTS];
    __shared__ int s_ulist[kSmallMaxSlots];
    __shared__ int s_uoff[kSmallMaxSlots + 1];
    __shared__ int s_ucur[kSmallMaxSlots];
    __shared__ int s_utok[kSmallMaxSlots];
    __shared__ int s_wcnt[32], s_wbase[32], s_U;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const int T = a.T, K = a.K, E = a.E, H = a.H, I = a.I, TK = T * K;
    pdl_wait();
    small_routing(a, s_ids, s_w, blockIdx.x == 0);
    for (int e = tid; e < E; e += blockDim.x) s_uidx[e] = -1;
    __syncthreads();
    for (int i = tid; i < TK; i += blockDim.x) s_uidx[s_ids[i]] = 0;
    __syncthreads();
    // distinct experts in ascending id order
    const int nchunk = cdiv(E, 32);
    for (int j = warp; j < nchunk; j += nw) {
        const int e = 32 * j + lane;
        const unsigned m = __ballot_sync(0xffffffffu, e < E && s_uidx[e] == 0);
        if (lane == 0) s_wcnt[j] = __popc(m);
    }
    __syncthreads();
    if (tid == 0) {
        int run = 0;
        for (int j = 0; j < nchunk; ++j) {
            s_wbase[j] = run;
            run += s_wcnt[j];
        }
        s_U = run;
    }
    __syncthreads();
    for (int j = warp; j < nchunk; j += nw) {
        const int e = 32 * j + lane;
        const bool f = e < E && s_uidx[e] == 0;
        const unsigned m = __ballot_sync(0xffffffffu, f);
        if (f) {
            const int u = s_wbase[j] + __popc(m & ((1u << lane) - 1u));
            s_ulist[u] = e;
            s_uidx[e] = u;
        }
    }
    __syncthreads();
    const int U = s_U;
    for (int u = tid; u < U; u += blockDim.x) s_ucur[u] = 0;
    __syncthreads();
    for (int i = tid; i < TK; i += blockDim.x) atomicAdd(&s_ucur[s_uidx[s_ids[i]]], 1);
    __syncthreads();
    if (warp == 0) {  // exclusive scan of the per-expert token counts
        int run = 0;
        for (int u0 = 0; u0 < U; u0 += 32) {
            const int u = u0 + lane;
            int v = (u < U) ? s_ucur[u] : 0;
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
    for (int u = tid; u < U; u += blockDim.x) s_ucur[u] = 0;
    __syncthreads();
    for (int i = tid; i < TK; i += blockDim.x) {
        const int t = i / K, k = i - t * K;
        const int u = s_uidx[s_ids[i]];
        s_utok[s_uoff[u] + atomicAdd(&s_ucur[u], 1)] = k * T + t;  // slot index
    }
    __syncthreads();
    pdl_trigger();

    // Bring the W2 rows the next kernel needs into L2 while this one streams W13: the
    // distinct experts' W2 matrices (contiguous [H, I] each) and the shared W2, split
    // evenly over the CTAs in 32 KB bulk prefetches.
    {
        const size_t per = (size_t)H * I * 2;
        const size_t tot = (size_t)U * per + (size_t)H * a.Is * 2;
        const size_t lo = tot * blockIdx.x / gridDim.x, hi = tot * (blockIdx.x + 1) / gridDim.x;
        const size_t lo16 = lo & ~(size_t)15, hi16 = (hi + 15) & ~(size_t)15;
        for (size_t off = lo16 + (size_t)tid * 32768; off < hi16; off += (size_t)blockDim.x * 32768) {
            const size_t end = off + 32768 < hi16 ? off + 32768 : hi16;
            const size_t u = off / per;
            if (u < (size_t)U) {
                const size_t uend = (u + 1) * per;
                const size_t stop = end < uend ? end : uend;
                bulk_prefetch_l2(reinterpret_cast<const uint8_t*>(a.w2 + (size_t)s_ulist[u] * H * I) + (off - u * per),
                                 (uint32_t)(stop - off));
            } else {
                const size_t so = off - (size_t)U * per;
                bulk_prefetch_l2(reinterpret_cast<const uint8_t*>(a.ws2) + so, (uint32_t)(end - off));
            }
        }
    }

    const int nch = H >> 3;
    const bool swiglu = a.act == MOE_ACT_SWIGLU;
    const long long Nr = (long long)U * I;
    const long long N = Nr + a.Is;
    const long long b0 = (long long)blockIdx.x * N / gridDim.x, b1 = (long long)(blockIdx.x + 1) * N / gridDim.x;
    for (long long item = b0 + warp; item < b1; item += nw) {
        const bf16* grow;
        const bf16* urow;
        const int* toks;
        int ntok, i, ld;
        bf16* outp;
        if (item < Nr) {
            const int u = (int)(item / I);
            i = (int)(item - (long long)u * I);
            const int e = s_ulist[u];
            const size_t rows = swiglu ? 2 * (size_t)I : (size_t)I;
            grow = a.w13 + ((size_t)e * rows + i) * H;
            urow = grow + (size_t)I * H;
            toks = s_utok + s_uoff[u];
            ntok = s_uoff[u + 1] - s_uoff[u];
            outp = a.h;
            ld = I;
        } else {
            i = (int)(item - Nr);
            grow = a.ws13 + (size_t)i * H;
            urow = grow + (size_t)a.Is * H;
            toks = nullptr;
            ntok = T;
            outp = a.hs;
            ld = a.Is;
        }
        uint4 wg[VH], wu[VH];
#pragma unroll
        for (int j = 0; j < VH; ++j) {
            const int c = lane + 32 * j;
            if (c < nch) {
                wg[j] = ld_stream16(grow + (size_t)c * 8);
                if (swiglu) wu[j] = ld_stream16(urow + (size_t)c * 8);
            }
        }
        for (int n = 0; n < ntok; ++n) {
            const int s = toks ? toks[n] : n;
            const int t = toks ? s % T : n;
            const bf16* xr = a.x + (size_t)t * H;
            float ag = 0.0f, au = 0.0f;
#pragma unroll
            for (int j = 0; j < VH; ++j) {
                const int c = lane + 32 * j;
                if (c < nch) {
                    const uint4 xv = ld_nc16(xr + (size_t)c * 8);
                    ag = dot8(wg[j], xv, ag);
                    if (swiglu) au = dot8(wu[j], xv, au);
                }
            }
            ag = warp_sum(ag);
            if (swiglu) au = warp_sum(au);
            if (lane == 0) {
                const float v = swiglu ? act_swiglu(ag, au) : act_relu2(ag);
                outp[(size_t)s * ld + i] = __float2bfloat16_rn(v);
            }
        }
    }
}

template <int VI>
__global__ void __launch_bounds__(256) fc2_small(const SmallArgs a) {
    __shared__ int s_ids[kSmallMaxSlots];
    __shared__ float s_w[kSmallMaxSlots];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const int T = a.T, K = a.K, H = a.H, I = a.I, Is = a.Is;
    // Routing again, from the same logits (complete before fc1 started): identical ids.
    small_routing(a, s_ids, s_w, false);
    __syncthreads();
    const int f0 = (int)((long long)blockIdx.x * H / gridDim.x);
    const int f1 = (int)((long long)(blockIdx.x + 1) * H / gridDim.x);
    const int nf = f1 - f0;
    pdl_wait();  // h from fc1 (W2 was prefetched into L2 by fc1)
    const int nchI = I >> 3, nchS = Is >> 3;
    // slots per batch: keep about 16 row chunks of W2 (and as many of h) in flight
    constexpr int KB = VI <= 2 ? 8 : (VI <= 4 ? 4 : (VI <= 8 ? 2 : 1));
    const int items = T * nf;
    for (int item = warp; item < items; item += nw) {
        const int t = item / nf, f = f0 + (item - t * nf);
        float acc = 0.0f;
        for (int k0 = 0; k0 < K; k0 += KB) {
            uint4 wv[KB][VI], hv[KB][VI];
#pragma unroll
            for (int kb = 0; kb < KB; ++kb) {
                const int k = k0 + kb;
                const bf16* row = a.w2 + ((size_t)(k < K ? s_ids[t * K + k] : 0) * H + f) * I;
                const bf16* hr = a.h + (size_t)((k < K ? k : 0) * T + t) * I;
#pragma unroll
                for (int j = 0; j < VI; ++j) {
                    const int c = lane + 32 * j;
                    if (k < K && c < nchI) {
                        wv[kb][j] = ld_nc16(row + (size_t)c * 8);
                        hv[kb][j] = ld_nc16(hr + (size_t)c * 8);
                    }
                }
            }
#pragma unroll
            for (int kb = 0; kb < KB; ++kb) {
                const int k = k0 + kb;
                if (k < K) {
                    float part = 0.0f;
#pragma unroll
                    for (int j = 0; j < VI; ++j)
                        if (lane + 32 * j < nchI) part = dot8(wv[kb][j], hv[kb][j], part);
                    acc = fmaf(s_w[t * K + k], part, acc);
                }
            }
        }
        const float routed = warp_sum(acc);
        float ys = 0.0f;
        if (Is) {
            const bf16* row = a.ws2 + (size_t)f * Is;
            const bf16* hr = a.hs + (size_t)t * Is;
            float part = 0.0f;
            for (int c = lane; c < nchS; c += 32)
                part = dot8(ld_nc16(row + (size_t)c * 8), ld_nc16(hr + (size_t)c * 8), part);
            ys = warp_sum(part);
        }
        if (lane == 0) {
            const float r = bf_round(routed);
            const float o = Is ? __fadd_rn(r, bf_round(ys)) : r;
            a.out[(size_t)t * H + f] = __float2bfloat16_rn(o);
        }
    }
    pdl_trigger();
}

static int pick_v(int chunks) {
    const int need = cdiv(chunks, 32);
    const int opts[] = {1, 2, 4, 8, 12, 16};
    for (int v : opts)
        if (v >= need) return v;
    return -1;
}

bool small_path_supported(int T, int H, int I, int Is) {
    return T <= kSmallMaxT && pick_v(H >> 3) > 0 && pick_v(I >> 3) > 0 && pick_v(Is >> 3) > 0;
}

cudaError_t launch_small(const SmallArgs& a, int num_sms, cudaStream_t s, bool pdl_first,
                         const std::function<bool()>* mark) {
    const int vh = pick_v(a.H >> 3), vi = pick_v(a.I >> 3);
    cudaError_t err = cudaErrorInvalidValue;
    dim3 block(256), g1(num_sms), g2(std::min(num_sms, a.H));
    const bool chain = mark == nullptr;
    if (mark && !(*mark)()) return cudaErrorUnknown;
#define MOE_F1(VV) \
    if (vh == VV) err = launch_k(fc1_small<VV>, g1, block, 0, s, pdl_first && chain, a);
    MOE_F1(1) MOE_F1(2) MOE_F1(4) MOE_F1(8) MOE_F1(12) MOE_F1(16)
#undef MOE_F1
    if (err != cudaSuccess) return err;
    err = cudaErrorInvalidValue;
    if (mark && !(*mark)()) return cudaErrorUnknown;
#define MOE_F2(VV) \
    if (vi == VV) err = launch_k(fc2_small<VV>, g2, block, 0, s, chain, a);
    MOE_F2(1) MOE_F2(2) MOE_F2(4) MOE_F2(8) MOE_F2(12) MOE_F2(16)
#undef MOE_F2
    return err;
}

}  // namespace moe
