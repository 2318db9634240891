// stream.cu -- the few-token path: only the routed experts' weights are read, each
// exactly once from HBM, by 16-byte coalesced loads spread over every SM.  Dot products
// run on the CUDA cores with warp-level XOR reductions; there is no split-K reduce
// kernel (the skinny-GEMM design of vLLM PR #64636, "Overview", applied to the routed
// experts).  The routing comes from the route table built once by route_small_kernel.
//
//   fc1_small: the (expert, feature) items -- a gate row and an up row of W13[e] (SwiGLU)
//              or a row of W1[e], and the shared expert's rows -- are split evenly over
//              one CTA per SM.  A producer thread streams the CTA's rows, kFc1Rows
//              consecutive rows of each half per stage, into a ring of shared-memory
//              stages with 1-D bulk copies; eight consumer warps dot each row with every
//              token routed to that expert (x staged in shared memory) and write
//              h[slot, i] = act(.) in BF16.  Before that, the consumers L2-prefetch the
//              CTA's share of the routed W2 for the next kernel.
//   fc2_small: each CTA owns a slice of output features f.  For every token it sums
//              w[t,k] * (W2[e_k, f, :] . h[slot]) in FP32 over the slots, scales the sum by
//              the routed scale, rounds to BF16, adds the BF16 shared-expert output (its
//              own, optionally gated, or the caller's) and rounds again ("MTP1 isolated
//              gather/shared-add closure": routed FP32 accumulation -> BF16 -> shared BF16
//              add -> BF16), writing the layer output directly.
#include <cstring>

#include "kernels.cuh"

namespace moe {

static constexpr int kSmallThreads = 512;  // fc2_small
static constexpr int kFc1Rows = 4;         // weight rows (of each half) per stage
static constexpr int kFc1Consumers = 8;    // consumer warps: two groups of kFc1Rows
static constexpr int kFc1Threads = 32 * (1 + kFc1Consumers);
static constexpr size_t kFc1SmemBudget = 200 * 1024;

struct Fc1Plan {  // host-side sizing of the stage ring
    int stages;
    size_t stage_bytes, x_bytes, smem;
};
static Fc1Plan fc1_plan(const SmallArgs& a) {
    Fc1Plan p;
    const int halves = a.act == MOE_ACT_SWIGLU ? 2 : 1;
    p.stage_bytes = (size_t)halves * kFc1Rows * a.H * 2;
    p.x_bytes = align_up((size_t)a.T * a.H * 2, 1024);
    const size_t avail = kFc1SmemBudget > p.x_bytes ? kFc1SmemBudget - p.x_bytes : 0;
    // Even: the two consumer groups take alternate stages, so with an even ring every slot
    // belongs to one group, which consumes its stages in order and therefore never waits
    // on a slot whose previous stage is still pending (an odd ring would let a group wait
    // for a phase parity that a fresh barrier reports as already complete).
    p.stages = (int)std::min<size_t>(8, avail / p.stage_bytes) & ~1;
    p.smem = 1024 + p.x_bytes + (size_t)p.stages * p.stage_bytes + 1024;
    return p;
}

// Walks a CTA's contiguous item range [b0, b1) in stages of up to kFc1Rows consecutive
// rows of one expert (or of the shared expert).
struct StageWalk {
    long long item, b1, Nr;
    int I, Is;
    __device__ bool next(int& u, int& i0, int& r) {
        if (item >= b1) return false;
        if (item < Nr) {
            u = (int)(item / I);
            i0 = (int)(item - (long long)u * I);
            r = (int)min((long long)min(kFc1Rows, I - i0), b1 - item);
        } else {
            u = -1;
            i0 = (int)(item - Nr);
            r = (int)min((long long)min(kFc1Rows, Is - i0), b1 - item);
        }
        item += r;
        return true;
    }
};

template <bool SWIGLU>
__global__ void __launch_bounds__(kFc1Threads, 1) fc1_small(const SmallArgs a, int stages, int stage_bytes,
                                                           int x_bytes) {
    __shared__ int s_ulist[kSmallMaxSlots];
    __shared__ int s_uoff[kSmallMaxSlots + 1];
    __shared__ int s_utok[kSmallMaxSlots];
    __shared__ __align__(8) uint64_t s_bar[2 * 8 + 1];  // full[8], empty[8], x
    __shared__ int s_abort;
    extern __shared__ uint8_t dsm[];
    const uint32_t raw = smem_u32(dsm);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* xsm = dsm + (base - raw);                 // x [T][H]
    const uint32_t ring = base + (uint32_t)x_bytes;    // stages
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int T = a.T, K = a.K, H = a.H, I = a.I, TK = T * K;
    const uint32_t bar0 = smem_u32(s_bar);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (8 + s); };
    const uint32_t x_bar = bar0 + 8u * 16;
    if (tid == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), kFc1Rows);
        }
        mbar_init(x_bar, 1);
        s_abort = 0;
        fence_mbar_init();
    }
    __syncthreads();
    pdl_wait();
    const RouteTable* rt = a.rt;
    const int U = rt->U;
    const long long Nr = (long long)U * I;
    const long long N = Nr + a.Is;
    const long long b0 = (long long)blockIdx.x * N / gridDim.x, b1 = (long long)(blockIdx.x + 1) * N / gridDim.x;
    const size_t rows1 = SWIGLU ? 2 * (size_t)I : (size_t)I;
    const uint32_t half_bytes = (uint32_t)kFc1Rows * H * 2;
    if (tid == 0) {  // x [T][H] in one bulk copy, ahead of the weight stream
        const uint32_t xb = (uint32_t)T * H * 2;
        mbar_expect_tx(x_bar, xb);
        bulk_copy_g2s(base, a.x, xb, x_bar);
    }
    if (warp != 0) {  // consumers stage the slot lists while the producer already streams
        for (int i = tid - 32; i < U; i += blockDim.x - 32) s_ulist[i] = rt->ulist[i];
        for (int i = tid - 32; i <= U; i += blockDim.x - 32) s_uoff[i] = rt->uoff[i];
        for (int i = tid - 32; i < TK; i += blockDim.x - 32) s_utok[i] = rt->utok[i];
        named_barrier(1, blockDim.x - 32);
    }
    pdl_trigger();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            StageWalk wk{b0, b1, Nr, I, a.Is};
            int u, i0, r, it = 0;
            while (wk.next(u, i0, r)) {
                const int s = it % stages;
                const uint32_t ph = (uint32_t)(it / stages) & 1u;
                if (!mbar_wait(empty_bar(s), ph ^ 1u, &s_abort, nullptr)) break;
                const bf16* g = (u >= 0) ? a.w13 + ((size_t)rt->ulist[u] * rows1 + i0) * H : a.ws13 + (size_t)i0 * H;
                const bf16* up = g + (size_t)((u >= 0) ? I : a.Is) * H;
                const uint32_t bytes = (uint32_t)r * H * 2;
                const uint32_t st = ring + (uint32_t)s * (uint32_t)stage_bytes;
                mbar_expect_tx(full_bar(s), SWIGLU ? 2 * bytes : bytes);
                bulk_copy_g2s(st, g, bytes, full_bar(s));
                if (SWIGLU) bulk_copy_g2s(st + half_bytes, up, bytes, full_bar(s));
                ++it;
            }
        }
    } else {
        // ------------------------------------------------------------ consumers
        // W2 of the routed experts and the shared W2 into L2 for the next kernel, split
        // evenly over the CTAs in 32 KB bulk prefetches.
        {
            const int ct = tid - 32;
            const size_t per = (size_t)H * I * 2;
            const size_t tot = (size_t)U * per + (size_t)H * a.Is * 2;
            const size_t lo = tot * blockIdx.x / gridDim.x, hi = tot * (blockIdx.x + 1) / gridDim.x;
            const size_t lo16 = lo & ~(size_t)15, hi16 = (hi + 15) & ~(size_t)15;
            for (size_t off = lo16 + (size_t)ct * 32768; off < hi16; off += (size_t)(blockDim.x - 32) * 32768) {
                const size_t end = off + 32768 < hi16 ? off + 32768 : hi16;
                const size_t u = off / per;
                if (u < (size_t)U) {
                    const size_t stop = end < (u + 1) * per ? end : (u + 1) * per;
                    bulk_prefetch_l2(reinterpret_cast<const uint8_t*>(a.w2 + (size_t)s_ulist[u] * H * I) + (off - u * per),
                                     (uint32_t)(stop - off));
                } else {
                    bulk_prefetch_l2(reinterpret_cast<const uint8_t*>(a.ws2) + (off - (size_t)U * per),
                                     (uint32_t)(end - off));
                }
            }
        }
        const int cw = warp - 1;
        const int grp = cw / kFc1Rows, row = cw % kFc1Rows;
        const int nch = H >> 3;
        StageWalk wk{b0, b1, Nr, I, a.Is};
        int u, i0, r, it = 0;
        const bool x_ok = mbar_wait(x_bar, 0, &s_abort, nullptr);
        while (x_ok && wk.next(u, i0, r)) {
            const int q = it++;
            if ((q & 1) != grp) continue;
            const int s = q % stages;
            const uint32_t ph = (uint32_t)(q / stages) & 1u;
            if (!mbar_wait(full_bar(s), ph, &s_abort, nullptr)) break;
            if (row < r) {
                const uint8_t* st = dsm + (ring - raw) + (size_t)s * stage_bytes;
                const uint4* grow = reinterpret_cast<const uint4*>(st + (size_t)row * H * 2);
                const uint4* urow = reinterpret_cast<const uint4*>(st + half_bytes + (size_t)row * H * 2);
                const int i = i0 + row;
                const int* toks = (u >= 0) ? s_utok + s_uoff[u] : nullptr;
                const int ntok = (u >= 0) ? s_uoff[u + 1] - s_uoff[u] : T;
                bf16* outp = (u >= 0) ? a.h : a.hs;
                const int ld = (u >= 0) ? I : a.Is;
                for (int n = 0; n < ntok; ++n) {
                    const int sl = toks ? toks[n] : n;
                    const int t = toks ? sl % T : n;
                    const uint4* xr = reinterpret_cast<const uint4*>(xsm + (size_t)t * H * 2);
                    float ag = 0.0f, au = 0.0f;
                    for (int c = lane; c < nch; c += 32) {
                        const uint4 xv = xr[c];
                        ag = dot8(grow[c], xv, ag);
                        if (SWIGLU) au = dot8(urow[c], xv, au);
                    }
                    ag = warp_sum(ag);
                    if (SWIGLU) au = warp_sum(au);
                    if (lane == 0) {
                        const float v = SWIGLU ? act_swiglu(ag, au) : act_relu2(ag);
                        outp[(size_t)sl * ld + i] = __float2bfloat16_rn(v);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty_bar(s));
        }
    }
    __syncthreads();
    if (s_abort) {  // a wait gave up: let bulk copies in flight land before the CTA retires
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 50000ull) {
        }
    }
}

template <int VI>
__global__ void __launch_bounds__(kSmallThreads, 1) fc2_small(const SmallArgs a) {
    __shared__ int s_ids[kSmallMaxSlots];
    __shared__ float s_w[kSmallMaxSlots];
    __shared__ float s_gate[kSmallMaxT];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const int T = a.T, K = a.K, H = a.H, I = a.I, Is = a.Is;
    const int f0 = (int)((long long)blockIdx.x * H / gridDim.x);
    const int f1 = (int)((long long)(blockIdx.x + 1) * H / gridDim.x);
    const int nf = f1 - f0;
    pdl_wait();  // h from fc1 (W2 is in L2 by now: fc1 prefetched it)
    for (int i = tid; i < T * K; i += blockDim.x) {
        s_ids[i] = a.rt->ids[i];
        s_w[i] = a.rt->w[i];
    }
    if (a.has_gate)
        for (int i = tid; i < T; i += blockDim.x) s_gate[i] = a.rt->gate[i];
    __syncthreads();
    const int nchI = I >> 3, nchS = Is >> 3;
    constexpr int KB = VI <= 2 ? 4 : (VI <= 4 ? 2 : 1);  // slots whose rows are in flight together
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
                    const bool ok = k < K && c < nchI;
                    wv[kb][j] = ok ? ld_nc16(row + (size_t)c * 8) : make_uint4(0u, 0u, 0u, 0u);
                    hv[kb][j] = ok ? ld_nc16(hr + (size_t)c * 8) : make_uint4(0u, 0u, 0u, 0u);
                }
            }
#pragma unroll
            for (int kb = 0; kb < KB; ++kb) {
                const int k = k0 + kb;
                if (k < K) {
                    float part = 0.0f;
#pragma unroll
                    for (int j = 0; j < VI; ++j) part = dot8(wv[kb][j], hv[kb][j], part);
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
            if (a.has_gate) ys = __fmul_rn(s_gate[t], ys);
        }
        if (lane == 0) {
            const float r = bf_round(__fmul_rn(a.routed_scale, routed));
            float o = r;
            if (Is) o = __fadd_rn(r, bf_round(ys));
            else if (a.sh_out) o = __fadd_rn(r, __bfloat162float(a.sh_out[(size_t)t * H + f]));  // read, then
            a.out[(size_t)t * H + f] = __float2bfloat16_rn(o);                                     // written in place
        }
    }
    pdl_trigger();
}

static int pick_v(int chunks) {
    const int need = cdiv(chunks, 32);
    const int opts[] = {1, 2, 4, 8, 10, 12, 16};
    for (int v : opts)
        if (v >= need) return v;
    return -1;
}

bool small_path_supported(int T, int H, int I, int Is) {
    if (T > kSmallMaxT || pick_v(I >> 3) <= 0 || pick_v(I >> 3) > 8) return false;
    SmallArgs a;
    std::memset(&a, 0, sizeof(a));
    a.T = T;
    a.H = H;
    a.act = MOE_ACT_SWIGLU;  // the larger stage
    return fc1_plan(a).stages >= 2;
}

cudaError_t launch_small(const SmallArgs& a, int num_sms, cudaStream_t s, bool pdl_first,
                         const std::function<bool()>* mark) {
    const int vi = pick_v(a.I >> 3);
    const Fc1Plan pl = fc1_plan(a);
    if (pl.stages < 2) return cudaErrorInvalidValue;
    cudaError_t err;
    dim3 block(kSmallThreads), g1(num_sms), g2(std::min(num_sms, a.H));
    const bool chain = mark == nullptr;
    if (mark && !(*mark)()) return cudaErrorUnknown;
    if (a.act == MOE_ACT_SWIGLU) {
        err = cudaFuncSetAttribute(fc1_small<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.smem);
        if (err == cudaSuccess)
            err = launch_k(fc1_small<true>, g1, dim3(kFc1Threads), pl.smem, s, pdl_first && chain, a, pl.stages,
                           (int)pl.stage_bytes, (int)pl.x_bytes);
    } else {
        err = cudaFuncSetAttribute(fc1_small<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.smem);
        if (err == cudaSuccess)
            err = launch_k(fc1_small<false>, g1, dim3(kFc1Threads), pl.smem, s, pdl_first && chain, a, pl.stages,
                           (int)pl.stage_bytes, (int)pl.x_bytes);
    }
    if (err != cudaSuccess) return err;
    err = cudaErrorInvalidValue;
    if (mark && !(*mark)()) return cudaErrorUnknown;
#define MOE_F2(VV) \
    if (vi == VV) err = launch_k(fc2_small<VV>, g2, block, 0, s, chain, a);
    MOE_F2(1) MOE_F2(2) MOE_F2(4) MOE_F2(8)
#undef MOE_F2
    return err;
}

}  // namespace moe
