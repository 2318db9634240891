// permute.cu -- group the M*K token slots by expert (FlashInfer PR #4646, walkthrough:
// routing permutation; review notes: count reduction, exclusive scan, per-expert
// offsets).  Unpadded.
//
// permute_kernel (the moe_permute entry point) is deterministic: within an expert, slots
// are in ascending token order.  permute_fast_kernel (inside moe_fused_forward) places
// slots with per-expert atomic cursors, so its order within an expert changes from run to
// run; its offsets and the set of slots of each expert do not.  Only the order of the FP32
// additions into the routed accumulator depends on it.
//
// permute_kernel: one CTA of 32 warps.  The tokens are split into 32 contiguous ranges, one per warp.
//   1. each warp histograms its range into its own row hist[w][e] (shared memory);
//   2. per expert, an exclusive scan down the 32 warp rows gives each warp's start
//      inside the expert; a block scan over experts gives the expert offsets;
//   3. each warp walks its tokens in order, lanes = slots (a token's experts are
//      distinct), and places slot k*M + t at offsets[e] + hist[w][e]++.
// It also writes the tile tables of the grouped GEMMs: for group g the number of
// 128-row token tiles times the feature tiles, as an exclusive prefix over groups.
#include "kernels.cuh"

namespace moe {
namespace {

constexpr int kThreads = 1024;

// Exclusive scan of one value per thread over the whole CTA; returns the total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* s_warp, int& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int w = s_warp[lane];
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += n;
        }
        s_warp[lane] = wi - w;
        if (lane == 31) s_warp[32] = wi;
    }
    __syncthreads();
    const int r = s_warp[warp] + incl - v;
    total = s_warp[32];
    __syncthreads();
    return r;
}

__device__ void write_tile_tables(const PermuteArgs& a, int my_cnt, int* s_warp);

__global__ void __launch_bounds__(kThreads, 1) permute_kernel(const PermuteArgs a) {
    extern __shared__ int smem[];
    const int E = a.E, M = a.M, K = a.K;
    int* hist = smem;               // [32][E]
    int* cnt = hist + 32 * E;       // [E]
    __shared__ int s_warp[33];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    pdl_wait();
    for (int i = tid; i < 32 * E; i += kThreads) hist[i] = 0;
    __syncthreads();
    const int chunk = cdiv(M, 32);
    const int t0 = min(M, warp * chunk), t1 = min(M, t0 + chunk);
    for (size_t i = (size_t)t0 * K + lane; i < (size_t)t1 * K; i += 32) {
        const int e = a.ids[i];
        if ((unsigned)e < (unsigned)E) atomicAdd(&hist[warp * E + e], 1);
        else set_dev_error(a.err, MOE_DEVERR_BAD_EXPERT_ID);
    }
    __syncthreads();
    for (int e = tid; e < E; e += kThreads) {
        int run = 0;
        for (int w = 0; w < 32; ++w) {
            const int v = hist[w * E + e];
            hist[w * E + e] = run;
            run += v;
        }
        cnt[e] = run;
    }
    __syncthreads();
    // expert offsets (E <= 1024 = one element per thread)
    int total;
    const int my_cnt = (tid < E) ? cnt[tid] : 0;
    const int off = block_exclusive_scan(my_cnt, s_warp, total);
    if (tid < E) a.offsets[tid] = off;
    if (tid == 0) a.offsets[E] = total;
    if (a.tiles1) write_tile_tables(a, my_cnt, s_warp);
    if (tid < E) {
        for (int w = 0; w < 32; ++w) hist[w * E + tid] += off;
    }
    __syncthreads();
    // stable scatter: warp w walks its tokens in order, 32 tokens per batch
    for (int tb = t0; tb < t1; tb += 32) {
        int ev[32];
#pragma unroll
        for (int j = 0; j < 32; ++j)
            ev[j] = (tb + j < t1 && lane < K) ? a.ids[(size_t)(tb + j) * K + lane] : -1;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int e = ev[j];
            if ((unsigned)e < (unsigned)E) {
                const int pos = atomicAdd(&hist[warp * E + e], 1);
                const int src = lane * M + tb + j;
                a.perm[pos] = src;
                if (a.inv) a.inv[src] = pos;
            }
        }
    }
    pdl_trigger();
}

// Tile tables of the grouped GEMMs from the per-expert counts (one thread per group).
__device__ void write_tile_tables(const PermuteArgs& a, int my_cnt, int* s_warp) {
    const int tid = threadIdx.x, E = a.E, M = a.M;
    const int G = E + (a.has_shared ? 1 : 0);
    const int rows = (tid < E) ? my_cnt : (tid == E && a.has_shared ? M : 0);
    const bool sh = tid == E;
    int tot1, tot2;
    const int p1 = block_exclusive_scan(tid < G ? cdiv(rows, a.bn1) * (sh ? a.nfeat1_s : a.nfeat1_r) : 0, s_warp, tot1);
    const int p2 = block_exclusive_scan(tid < G ? cdiv(rows, a.bn2) * (sh ? a.nfeat2_s : a.nfeat2_r) : 0, s_warp, tot2);
    if (tid < G) {
        a.tiles1[tid] = p1;
        a.tiles2[tid] = p2;
    }
    if (tid == 0) {
        a.tiles1[G] = tot1;
        a.tiles2[G] = tot2;
    }
}

// Every CTA scans the counts into offsets (E <= 1024 values); CTA 0 also publishes the
// offsets and the tile tables; each thread then places one slot.  The order of the slots
// within an expert's segment is unspecified (CTA and atomic arrival order).
__global__ void __launch_bounds__(kThreads) permute_fast_kernel(const PermuteArgs a, const int* __restrict__ counts,
                                                               int* __restrict__ cursor) {
    __shared__ int s_off[MOE_MAX_EXPERTS];
    __shared__ int s_cnt[MOE_MAX_EXPERTS];   // this CTA's slots per expert
    __shared__ int s_base[MOE_MAX_EXPERTS];  // this CTA's first position inside each expert
    __shared__ int s_warp[33];
    const int tid = threadIdx.x, E = a.E;
    pdl_wait();
    const long long i = (long long)blockIdx.x * kThreads + tid;
    const bool has = i < (long long)a.M * a.K;
    const int e = has ? a.ids[i] : -1;  // issued before the scan, so its latency overlaps it
    const int my_cnt = (tid < E) ? counts[tid] : 0;
    if (tid < E) s_cnt[tid] = 0;  // ordered before the counting below by the scan's barriers
    int total;
    const int off = block_exclusive_scan(my_cnt, s_warp, total);
    if (tid < E) s_off[tid] = off;
    if (blockIdx.x == 0) {
        if (tid < E) a.offsets[tid] = off;
        if (tid == 0) a.offsets[E] = total;
        if (a.tiles1) write_tile_tables(a, my_cnt, s_warp);
    }
    // Rank of the slot among this CTA's slots of the same expert, then one global atomic
    // per (CTA, expert) reserves the CTA's contiguous range inside the expert's segment.
    const bool ok = has && (unsigned)e < (unsigned)E;
    const int local = ok ? atomicAdd(&s_cnt[e], 1) : 0;
    __syncthreads();
    if (tid < E) s_base[tid] = s_cnt[tid] > 0 ? atomicAdd(cursor + tid, s_cnt[tid]) : 0;
    __syncthreads();
    if (ok) {
        const int t = (int)(i / a.K), k = (int)(i - (long long)t * a.K);
        const int pos = s_off[e] + s_base[e] + local;
        if ((unsigned)pos < (unsigned)(a.M * a.K)) {
            a.perm[pos] = k * a.M + t;
            if (a.inv) a.inv[k * a.M + t] = pos;
        } else {  // the counts disagree with the ids: flag it, place nothing out of range
            set_dev_error(a.err, MOE_DEVERR_BAD_INDEX);
        }
    } else if (has) {
        set_dev_error(a.err, MOE_DEVERR_BAD_EXPERT_ID);
    }
    pdl_trigger();
}

}  // namespace

cudaError_t launch_permute_fast(const PermuteArgs& a, const int* counts, int* cursor, cudaStream_t s, bool pdl) {
    const long long n = (long long)a.M * a.K;
    const int grid = (int)std::max<long long>(1, (n + kThreads - 1) / kThreads);
    return launch_k(permute_fast_kernel, dim3(grid), dim3(kThreads), 0, s, pdl, a, counts, cursor);
}

size_t permute_smem_bytes(int E) { return (size_t)(33 * E) * sizeof(int); }

cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t s, bool pdl) {
    const size_t smem = permute_smem_bytes(a.E);
    cudaError_t e = cudaFuncSetAttribute(permute_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_k(permute_kernel, dim3(1), dim3(kThreads), smem, s, pdl, a);
}

}  // namespace moe
