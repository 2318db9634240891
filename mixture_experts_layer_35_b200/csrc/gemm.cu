// gemm.cu -- grouped BF16 GEMMs of the many-token path on the 5th-generation tensor
// cores (tcgen05.mma, FP32 accumulators in TMEM), and the finalize kernel.
//
// Orientation ("swap AB"): the MMA's M side is 128 output features of one expert's
// weight matrix, its N side is up to 128 routed token rows of that expert, so a tile's
// MMA N is the expert's actual row count rounded up to 16 (no padding to 128 when an
// expert receives few tokens).  K runs over the reduction dimension in 64-element steps
// (one 128-byte swizzle row of BF16).
//
//   FC1 (FlashInfer PR #4646 walkthrough: grouped BF16 GEMM + activation): A = W13[e]
//       rows of 128 features (SwiGLU: the gate and up halves as two accumulators), B =
//       the expert's tokens gathered row by row from x with cp.async into the swizzled
//       layout; epilogue applies SwiGLU / ReLU^2 and stores h (BF16) in permuted order.
//   FC2: A = W2[e] rows of 128 output features, B = the expert's contiguous h rows
//       (TMA, 32-row boxes); epilogue scales by the routing weight, transposes 4x4 blocks
//       within groups of 4 lanes and adds into the FP32 accumulator acc[t, :] with 16-byte
//       vector reductions, 4 consecutive features of one token per lane ("weighted output
//       combination").
//       The shared expert is one more group whose FC2 output is rounded to BF16 into ys.
//   DENSE: router logits, A = Wr (128 experts per tile), B = x rows (TMA).  It reads
//       nothing an earlier kernel of the call writes, so it waits on the previous kernel
//       (the call's prep kernel) only at its end and overlaps it.
//
// Warp roles (one CTA per SM, persistent over a group-major tile list):
//   warp 0      TMA producer (weights; FC2/DENSE token rows)
//   warp 1      TMEM allocator and single-thread MMA issuer
//   warps 2-    epilogue: tcgen05.ld of the accumulator (warp w reads TMEM lanes of
//               quarter w % 4), activation / scaling, stores.  Four warps, or with
//               wide tiles eight (FC1) or twelve (FC2): the warps of a quarter take
//               32-token column chunks in turn
//   then        FC1 only: eight warps gathering token rows of x with cp.async
// Shared memory holds a ring of stages (full/empty mbarriers); TMEM holds two
// accumulator buffers so the epilogue of one tile overlaps the mainloop of the next.
#include "kernels.cuh"

namespace moe {
namespace {

constexpr int BM = 128, BK = 64;
constexpr int A_BYTES = BM * BK * 2;  // 16 KB
// Token rows per TMA box of the B operand: FC2's h rows come in 32-row boxes (half the
// copies per stage of 16-row boxes; measured -18 % on FC2 at 192 rows per expert), the
// router's x rows in 16-row boxes.  A box may run past the tile's rows: the MMA reads
// only the tile's rows rounded up to 16, so the extra rows are never used.
template <int MODE>
__host__ __device__ constexpr int b_box_rows() {
    return MODE == GM_FC2 ? kFc2BoxRows : 16;
}

template <int MODE, int BN>
struct Cfg {
    static constexpr bool kGather = (MODE == GM_FC1_SWIGLU || MODE == GM_FC1_RELU2);
    static constexpr bool kSwiglu = (MODE == GM_FC1_SWIGLU);
    static constexpr int kNA = kSwiglu ? 2 : 1;
    static constexpr int kBN = BN;
    static constexpr int kBBytes = kBN * BK * 2;
    static constexpr int kStageBytes = kNA * A_BYTES + kBBytes;
    // Epilogue warps: FC2's epilogue (weighting, transposes, vector reductions) is heavy
    // next to its short mainloop, so with wide tiles it gets three warps per TMEM lane
    // quarter, splitting the token columns (measured at T = 4096 / 8192 of the
    // Qwen3.6-shaped layer, FC2: 4 warps 240 / 582 us, 8 warps 144 / 322 us, 12 warps
    // 137 / 276 us, 16 warps 140 / 304 us).  FC1 with tiles of 128+ tokens gets two
    // per quarter (together with 8 gather warps: FC1 244 -> 227 us at T = 4096).
    static constexpr int kEpiWarps =
        (MODE == GM_FC2 && BN > 32) ? 12 : ((kGather && BN >= 128) ? 8 : 4);
    static constexpr int kEpiBytes = 0;  // epilogues work from registers
    static constexpr int kAccCols = kSwiglu ? 2 * kBN : kBN;
    // Two accumulator buffers (the epilogue of one tile overlaps the next mainloop) when
    // they fit TMEM's 512 columns; a 256-token SwiGLU tile (gate + up = 512 columns) has one.
    static constexpr int kAccBufs = (2 * kAccCols) <= 512 ? 2 : 1;
    // Buffer stride in TMEM columns, padded to a multiple of 64.
    static constexpr int kAccStride = (kAccCols + 63) / 64 * 64;
    static constexpr int kTmemCols =
        (kAccBufs * kAccStride) > 256 ? 512 : ((kAccBufs * kAccStride) > 128 ? 256 : 128);
    static_assert(kAccBufs * kAccStride <= 512 || kAccBufs == 1, "accumulator buffers exceed TMEM");
    static_assert(kAccCols <= 512, "accumulator exceeds TMEM");
    // FC1 gather warps: each thread copies one 16-byte chunk (of 8 per 128-byte row) of
    // every kGatherRowStep-th token row of a stage.  Eight warps keep more rows in flight
    // than four (FC1 at T = 4096 of the Qwen3.6-shaped layer: 244 -> 235 us alone).
    static constexpr int kGatherWarps = kGather ? 8 : 0;
    static constexpr int kGatherThreads = 32 * kGatherWarps;
    static constexpr int kGatherRowStep = kGather ? kGatherThreads / 8 : 16;  // (unused without a gather)
    static_assert(!kGather || kBN % kGatherRowStep == 0, "gather rows must tile the token tile");
    static constexpr int kThreads = 64 + 32 * kEpiWarps + kGatherThreads;
    // FC1 gather: stages of token rows in flight before the gather warps signal the oldest
    // one.  It must stay at most kStages - 2: the gather can only issue stage j + lag once
    // the MMA has freed that slot, so with lag = kStages - 1 the signal for stage j waits
    // for the MMA to finish stage j - 1 and every stage starts late (measured: lag 3 of 4
    // stages, and lag 2 of 3, both stall; one warp per stage is slower too).
    static constexpr int kLagMax = 2;
    static constexpr int kMaxGroups = MOE_MAX_EXPERTS + 1;
    // Dynamic schedule: a ring of tile ids from the producer to the other roles.
    static constexpr int kIdSlots = 8;
    static constexpr int kIdConsumers = 1 + kEpiWarps + kGatherWarps;  // MMA thread, warps
    static constexpr size_t kRingOff = 256 + (size_t)(kMaxGroups + 1) * 4 * 2 + 64;
    static constexpr size_t kMeta = kRingOff + (size_t)kIdSlots * (8 + 8 + 4) + 64;
    // As many stages as the 227 KB of shared memory hold (at most 12: the barrier block).
    static constexpr int kStages =
        (int)((227 * 1024 - 1024 - kMeta - kEpiBytes) / kStageBytes) < 12
            ? (int)((227 * 1024 - 1024 - kMeta - kEpiBytes) / kStageBytes)
            : 12;
    // dynamic smem: alignment slack, stages, barriers, flags, tile and offset tables
    static constexpr size_t kSmem = 1024 + (size_t)kStages * kStageBytes + kEpiBytes + kMeta;
    static constexpr int kLag = (kStages - 2) < kLagMax ? (kStages - 2) : kLagMax;
    static_assert(kStages >= 3, "ring too shallow");
    static_assert(kGather || kBN % b_box_rows<MODE>() == 0, "a tile's boxes must fit its stage");
    static_assert(8 * (2 * kStages + 4) + 8 <= 256, "barrier block");
};

struct TileInfo {
    int g, ft, n, row0, shared;
    int nk;    // k-blocks of this tile
    int ntok;  // token tiles of this group (each streams the group's weight slice)
};

template <int BN>
__device__ __forceinline__ TileInfo decode_tile(const GemmArgs& a, const int* s_tiles, const int* s_offs, int G,
                                                int tile) {
    TileInfo ti;
    if (a.dense) {  // tile = (feature tile, token tile), token tile fastest
        const int ntok = cdiv(a.T, kDenseTokenTile);
        ti.g = 0;
        ti.ft = tile / ntok;
        const int tt = tile - ti.ft * ntok;
        ti.row0 = tt * kDenseTokenTile;
        ti.n = min(kDenseTokenTile, a.T - ti.row0);
        ti.shared = 0;
        ti.nk = cdiv(a.kdim, BK);
        ti.ntok = ntok;
        return ti;
    }
    int lo = 0, hi = G;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_tiles[mid] <= tile) lo = mid;
        else hi = mid;
    }
    const int g = lo;
    const int local = tile - s_tiles[g];
    const bool sh = a.has_shared && g == a.E;
    const int rows = sh ? a.T : (s_offs[g + 1] - s_offs[g]);
    const int ntok = cdiv(rows, BN);
    ti.g = g;
    ti.ft = local / ntok;
    const int tt = local - ti.ft * ntok;
    ti.row0 = (sh ? 0 : s_offs[g]) + tt * BN;
    ti.n = min(BN, rows - tt * BN);
    ti.shared = sh;
    ti.nk = cdiv(sh ? a.kdim_s : a.kdim, BK);
    ti.ntok = ntok;
    if (ti.n <= 0 || ti.row0 < 0) {  // only from corrupted tables: every role skips the tile
        set_dev_error(a.err, MOE_DEVERR_BAD_INDEX);
        ti.n = 0;
        ti.nk = 0;
    }
    return ti;
}

// One unit of a CTA's work: a whole tile, or (stream-K) a contiguous range of its k-blocks.
enum SegKind { kWhole = 0, kFixer = 1, kPart = 2 };
struct Seg {
    int tile, kb0, kb1;
    int kind;  // kWhole; kFixer: holds the tile's first k-blocks and adds the other CTAs' partial
               // sums before the epilogue (FC1); kPart: a later k-block range (FC1: its partial
               // sum goes to this CTA's scratch slot; FC2: reduced into the accumulator directly)
    int last;  // kFixer: last CTA whose range holds k-blocks of this tile
};

// A CTA's work.  Without stream-K, tiles are dealt round-robin.  With stream-K (few tiles
// for the grid: one wave or a few, where whole tiles would leave SMs idle at the end),
// the iteration space -- every tile's k-blocks, tiles in group-major order, routed tiles
// with nk_r k-blocks and the shared group's with nk_s -- is split into gridDim.x equal
// contiguous ranges, cut at tile boundaries into segments.  Every role of the CTA walks
// the same sequence.
template <bool SK>
struct WorkWalk {
    int total, R, nk_r, nk_s, streamk, next_tile;
    long long N, hi, i;
    __device__ void init(int total_, int R_, int nk_r_, int nk_s_, bool sk) {
        total = total_;
        R = R_;
        nk_r = nk_r_;
        nk_s = nk_s_;
        streamk = (SK && sk) ? 1 : 0;
        N = (long long)R * nk_r + (long long)(total - R) * nk_s;
        i = lo_of(blockIdx.x);
        hi = lo_of(blockIdx.x + 1);
        next_tile = blockIdx.x;
    }
    __device__ long long lo_of(int b) const { return N * b / gridDim.x; }
    // CTA whose range holds iteration it: the largest b with lo_of(b) <= it.
    __device__ int owner(long long it) const { return (int)(((it + 1) * gridDim.x - 1) / N); }
    __device__ bool next(Seg& s) {
        if (!SK || !streamk) {
            if (next_tile >= total) return false;
            s.tile = next_tile;
            s.kb0 = 0;
            s.kb1 = next_tile < R ? nk_r : nk_s;
            s.kind = kWhole;
            s.last = blockIdx.x;
            next_tile += gridDim.x;
            return true;
        }
        if (i >= hi) return false;
        const long long rr = (long long)R * nk_r;
        long long tb;
        int nk;
        if (i < rr) {
            s.tile = (int)(i / nk_r);
            tb = (long long)s.tile * nk_r;
            nk = nk_r;
        } else {
            const int j = (int)((i - rr) / nk_s);
            s.tile = R + j;
            tb = rr + (long long)j * nk_s;
            nk = nk_s;
        }
        const long long end = hi < tb + nk ? hi : tb + nk;
        s.kb0 = (int)(i - tb);
        s.kb1 = (int)(end - tb);
        s.kind = (s.kb0 == 0 && s.kb1 == nk) ? kWhole : (s.kb0 == 0 ? kFixer : kPart);
        s.last = s.kind == kFixer ? owner(tb + nk - 1) : (int)blockIdx.x;
        i = end;
        return true;
    }
    // CTA c holds iterations (its range is not empty).
    __device__ bool active(int c) const { return lo_of(c) < lo_of(c + 1); }
};

// FC2 epilogue of one 32-column chunk (see the comment at its call).
__device__ __forceinline__ void combine_chunk(const uint32_t (&v)[32], int mt, float mw, int c0, int n, int f,
                                              int feat, int T, float* __restrict__ acc, int lane) {
    const int i4 = lane & 3;
    const bool fok4 = f - i4 + 3 < feat;  // features of my group (feat % 8 == 0)
#pragma unroll
    for (int j0 = 0; j0 < 32; j0 += 4) {
        float r[4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) r[jj] = __uint_as_float(v[j0 + jj]);
        // r[jj] = y[feature of this lane, token j0 + jj]; 4x4 transpose
        float t0 = (i4 & 1) ? r[0] : r[1], t1 = (i4 & 1) ? r[2] : r[3];
        t0 = __shfl_xor_sync(0xffffffffu, t0, 1);
        t1 = __shfl_xor_sync(0xffffffffu, t1, 1);
        if (i4 & 1) {
            r[0] = t0;
            r[2] = t1;
        } else {
            r[1] = t0;
            r[3] = t1;
        }
        float u0 = (i4 & 2) ? r[0] : r[2], u1 = (i4 & 2) ? r[1] : r[3];
        u0 = __shfl_xor_sync(0xffffffffu, u0, 2);
        u1 = __shfl_xor_sync(0xffffffffu, u1, 2);
        if (i4 & 2) {
            r[0] = u0;
            r[1] = u1;
        } else {
            r[2] = u0;
            r[3] = u1;
        }
        const int tok = __shfl_sync(0xffffffffu, mt, j0 + i4);
        const float wt = __shfl_sync(0xffffffffu, mw, j0 + i4);
        if (c0 + j0 + i4 < n && fok4 && (unsigned)tok < (unsigned)T)
            red_add_v4_f32(acc + (size_t)tok * feat + (f - i4), wt * r[0], wt * r[1], wt * r[2], wt * r[3]);
    }
}

// Whole tiles dealt round-robin over persistent CTAs (every call except few-token ones,
// which take gemm_sk_kernel below).
// DYN: dynamic tile schedule.  After a round-robin prefix, the producer thread takes each
// next tile from a device counter (atomicAdd) when its ring is ready for one, and passes
// every id through a ring of kIdSlots shared-memory slots (mbarriers full/empty) to the MMA
// thread, the epilogue warps and the gather warps, which take the ids in the same order.
// The id after the last tile (>= total) ends every role's loop.  Without DYN, all tiles
// are dealt round-robin.
template <int MODE, int BN, bool DYN>
__global__ void __launch_bounds__(Cfg<MODE, BN>::kThreads, 1)
    gemm_kernel(const GemmArgs a, const __grid_constant__ CUtensorMap tm_a_r, const __grid_constant__ CUtensorMap tm_a_s,
                const __grid_constant__ CUtensorMap tm_b_r, const __grid_constant__ CUtensorMap tm_b_s) {
    using C = Cfg<MODE, BN>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t base_u32 = (raw_u32 + 1023u) & ~1023u;
    uint8_t* base = smem_raw + (base_u32 - raw_u32);
    uint8_t* meta = base + (size_t)C::kStages * C::kStageBytes + C::kEpiBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(meta);  // full[S], empty[S], tfull[2], tempty[2]
    const uint32_t bar_u32 = smem_u32(bars);
    auto full_bar = [&](int s) { return bar_u32 + 8u * s; };
    auto empty_bar = [&](int s) { return bar_u32 + 8u * (C::kStages + s); };
    auto tfull_bar = [&](int b) { return bar_u32 + 8u * (2 * C::kStages + b); };
    auto tempty_bar = [&](int b) { return bar_u32 + 8u * (2 * C::kStages + 2 + b); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(meta + 8 * (2 * C::kStages + 4));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* s_tiles = reinterpret_cast<int*>(meta + 256);
    int* s_offs = s_tiles + C::kMaxGroups + 1;
    // tile-id ring (DYN): full[kIdSlots], empty[kIdSlots], ids[kIdSlots]
    const uint32_t ring_u32 = smem_u32(meta + C::kRingOff);
    auto idfull_bar = [&](int j) { return ring_u32 + 8u * j; };
    auto idempty_bar = [&](int j) { return ring_u32 + 8u * (C::kIdSlots + j); };
    volatile int* s_ids = reinterpret_cast<volatile int*>(meta + C::kRingOff + 16 * C::kIdSlots);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = a.E + (a.has_shared ? 1 : 0);
    // Phase trace (optional): this CTA's row of the kernel's trace block.
    unsigned long long* trow = a.trace ? a.trace + (size_t)blockIdx.x * MOE_TRACE_FIELDS : nullptr;
    if (trow && threadIdx.x == 0) trow[MOE_TRACE_ENTRY] = globaltimer_ns();

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(full_bar(s), 1 + C::kGatherThreads);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), C::kEpiWarps);
        }
        if (DYN) {
            for (int j = 0; j < C::kIdSlots; ++j) {
                mbar_init(idfull_bar(j), 1);
                mbar_init(idempty_bar(j), C::kIdConsumers);
            }
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_a_r);
        if (a.has_shared) tma_prefetch_desc(&tm_a_s);
        if (!C::kGather) {
            tma_prefetch_desc(&tm_b_r);
            if (a.has_shared) tma_prefetch_desc(&tm_b_s);
        }
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);

    // Everything below reads what earlier kernels wrote (tile tables, perm, h) -- except
    // in DENSE mode, which reads only the caller's x and Wr and waits at its end.
    if (MODE != GM_DENSE) pdl_wait();
    if (!a.dense) {
        for (int i = threadIdx.x; i <= G; i += blockDim.x) s_tiles[i] = a.tiles[i];
        for (int i = threadIdx.x; i <= a.E; i += blockDim.x) s_offs[i] = a.offsets[i];
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (trow && threadIdx.x == 0) trow[MOE_TRACE_READY] = globaltimer_ns();
    const uint32_t tmem_base = *tmem_slot;
    const int total = a.dense ? a.nfeat_r * cdiv(a.T, kDenseTokenTile) : s_tiles[G];
    // Tiles are dealt round-robin over the persistent CTAs: at any moment the CTAs work on
    // neighbouring tiles of the group-major list (one expert's feature and token tiles),
    // which share that expert's weight rows and token rows in L2, and tiles of unequal
    // cost (ragged token tails) spread evenly.  The dynamic schedule takes the tiles in
    // the same list order, each from the first producer that is ready for one.
    int dj = 0;  // DYN: this role's position in the tile-id ring
    // The first three quarters of the rounds (all but at least two) stay round-robin, so
    // that neighbouring tiles still run side by side; the rest go to whichever CTA is
    // ready first.
    const int rr_rounds = DYN ? max(0, (3 * cdiv(total, (int)gridDim.x)) / 4 - 1) : 0;
    // Producer: the next tile (round-robin prefix, then the counter), published to the
    // ring (>= total: the end).
    auto id_produce = [&]() -> int {
        const int slot = dj % C::kIdSlots;
        const uint32_t ph = (uint32_t)(dj / C::kIdSlots) & 1u;
        if (!mbar_wait(idempty_bar(slot), ph ^ 1u, abort_flag, a.err)) return total;
        int t = dj < rr_rounds ? (int)blockIdx.x + dj * (int)gridDim.x
                                : rr_rounds * (int)gridDim.x + atomicAdd(a.dyn_ctr, 1);
        if (t > total) t = total;
        s_ids[slot] = t;
        mbar_arrive(idfull_bar(slot));
        ++dj;
        return t;
    };
    // Consumer (one thread, or every lane of a warp with `warp_wide`): the next id.
    auto id_consume = [&](bool warp_wide) -> int {
        const int slot = dj % C::kIdSlots;
        const uint32_t ph = (uint32_t)(dj / C::kIdSlots) & 1u;
        if (!mbar_wait(idfull_bar(slot), ph, abort_flag, a.err)) return total;
        const int t = s_ids[slot];
        ++dj;
        if (warp_wide) __syncwarp();
        if (!warp_wide || lane == 0) mbar_arrive(idempty_bar(slot));
        return t;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t wpol = l2_policy_evict_first();
            int it = 0, ntiles = 0;
            for (int tile = DYN ? id_produce() : (int)blockIdx.x; tile < total && !*abort_flag;
                 tile = DYN ? id_produce() : tile + (int)gridDim.x) {
                ++ntiles;
                const TileInfo ti = decode_tile<C::kBN>(a, s_tiles, s_offs, G, tile);
                const bool sh = ti.shared;
                const CUtensorMap* ta = sh ? &tm_a_s : &tm_a_r;
                const CUtensorMap* tb = sh ? &tm_b_s : &tm_b_r;
                const int frow = ti.ft * BM;
                constexpr int BBOX = b_box_rows<MODE>();
                const int nbox = cdiv(ti.n, BBOX);
                const uint32_t bytes = C::kNA * A_BYTES + (C::kGather ? 0u : (uint32_t)nbox * BBOX * BK * 2);
                for (int kb = 0; kb < ti.nk; ++kb, ++it) {
                    const int s = it % C::kStages;
                    const uint32_t ph = (uint32_t)(it / C::kStages) & 1u;
                    if (!mbar_wait(empty_bar(s), ph ^ 1u, abort_flag, a.err)) break;
                    const uint32_t st = base_u32 + (uint32_t)s * C::kStageBytes;
                    mbar_expect_tx(full_bar(s), bytes);
                    if (sh || a.dense) {
                        tma_load_2d(st, ta, full_bar(s), kb * BK, frow);
                        if (C::kSwiglu) tma_load_2d(st + A_BYTES, ta, full_bar(s), kb * BK, a.up_s + frow);
                    } else if (MODE == GM_FC2 || ti.ntok == 1) {
                        // Weights that no other tile of this call reads: evict first, so that
                        // they do not push the token rows, h and the accumulator out of L2
                        // (measured on FC1: -9 % at 16 tokens, -6 % at 4096 tokens of the
                        // Qwen3.6-shaped layer).
                        tma_load_3d_hint(st, ta, full_bar(s), kb * BK, frow, ti.g, wpol);
                        if (C::kSwiglu)
                            tma_load_3d_hint(st + A_BYTES, ta, full_bar(s), kb * BK, a.up_r + frow, ti.g, wpol);
                    } else {  // a second token tile of this expert streams the same slice
                        tma_load_3d(st, ta, full_bar(s), kb * BK, frow, ti.g);
                        if (C::kSwiglu) tma_load_3d(st + A_BYTES, ta, full_bar(s), kb * BK, a.up_r + frow, ti.g);
                    }
                    if (!C::kGather) {
                        const uint32_t bs = st + C::kNA * A_BYTES;
                        for (int q = 0; q < nbox; ++q)
                            tma_load_2d(bs + (uint32_t)q * (BBOX * BK * 2), tb, full_bar(s), kb * BK,
                                        ti.row0 + q * BBOX);
                    }
                }
            }
            if (trow) {
                trow[MOE_TRACE_LOADS_DONE] = globaltimer_ns();
                trow[MOE_TRACE_UNITS] = (unsigned long long)ntiles;
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int it = 0, tcount = 0;
            for (int tile = DYN ? id_consume(false) : (int)blockIdx.x; tile < total && !*abort_flag;
                 tile = DYN ? id_consume(false) : tile + (int)gridDim.x, ++tcount) {
                const TileInfo ti = decode_tile<C::kBN>(a, s_tiles, s_offs, G, tile);
                const int nk = ti.nk;
                const int npad = cdiv(ti.n, 16) * 16;
                const uint32_t idesc = idesc_bf16_f32(BM, npad);
                const int buf = tcount % C::kAccBufs;
                const uint32_t tph = (uint32_t)(tcount / C::kAccBufs) & 1u;
                if (!mbar_wait(tempty_bar(buf), tph ^ 1u, abort_flag, a.err)) break;
                tc_fence_after();
                const uint32_t d0 = tmem_base + (uint32_t)(buf * C::kAccStride);
                const uint32_t d1 = d0 + C::kBN;
                bool ok = true;
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % C::kStages;
                    const uint32_t ph = (uint32_t)(it / C::kStages) & 1u;
                    if (!mbar_wait(full_bar(s), ph, abort_flag, a.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = base_u32 + (uint32_t)s * C::kStageBytes;
                    const uint32_t bsm = st + C::kNA * A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint32_t accum = (kb > 0 || kk > 0) ? 1u : 0u;
                        const uint64_t bdesc = sdesc_sw128(bsm + kk * 32);
                        tc_mma(d0, sdesc_sw128(st + kk * 32), bdesc, idesc, accum);
                        if (C::kSwiglu) tc_mma(d1, sdesc_sw128(st + A_BYTES + kk * 32), bdesc, idesc, accum);
                    }
                    tc_commit(empty_bar(s));
                }
                if (!ok) break;
                tc_commit(tfull_bar(buf));
            }
        }
    } else if (warp < 2 + C::kEpiWarps) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                     // TMEM lane quarter of this warp
        const int half = (warp - 2) >> 2;          // FC2: which token columns (chunk parity)
        const int nhalf = C::kEpiWarps / 4;
        const int et = threadIdx.x - 64;
        if (a.zero_ptr) {
            float4* z = reinterpret_cast<float4*>(a.zero_ptr);
            const size_t n4 = a.zero_n / 4;
            const int ne = 32 * C::kEpiWarps;
            for (size_t i = (size_t)blockIdx.x * ne + et; i < n4; i += (size_t)gridDim.x * ne)
                z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        int tcount = 0;
        // (the abort flag is checked through the per-tile wait below)
        // 32-token chunks per half of the epilogue warps (the last may lie past the tile)
        constexpr int kChunks = (C::kBN + 32 * (C::kEpiWarps / 4) - 1) / (32 * (C::kEpiWarps / 4));
        for (int tile = DYN ? id_consume(true) : (int)blockIdx.x; tile < total;
             tile = DYN ? id_consume(true) : tile + (int)gridDim.x, ++tcount) {
            const TileInfo ti = decode_tile<C::kBN>(a, s_tiles, s_offs, G, tile);
            const int buf = tcount % C::kAccBufs;
            const uint32_t tph = (uint32_t)(tcount / C::kAccBufs) & 1u;
            // FC2: token and routing weight of each column this thread will scale, loaded
            // before the accumulator is ready (hidden behind the tile's mainloop).
            int mt[kChunks];
            float mw[kChunks];
#pragma unroll
            for (int ci = 0; ci < kChunks; ++ci) {
                mt[ci] = 0;
                mw[ci] = 0.0f;
                const int colm = 32 * half + 32 * nhalf * ci + lane;
                if (MODE == GM_FC2 && !ti.shared && colm < ti.n && ti.row0 + ti.n <= a.T * a.K) {
                    const int src = a.perm[ti.row0 + colm];
                    if ((unsigned)src < (unsigned)(a.T * a.K)) {
                        const int kk = src / a.T;
                        mt[ci] = src - kk * a.T;
                        mw[ci] = a.topk_w[(size_t)mt[ci] * a.K + kk];
                    } else {  // never from a valid permutation: flag it, contribute nothing
                        set_dev_error(a.err, MOE_DEVERR_BAD_INDEX);
                    }
                }
            }
            const bool waited = mbar_wait(tfull_bar(buf), tph, abort_flag, a.err);
            if (!waited) break;
            tc_fence_after();
            // The tile's rows must lie inside their buffer (they do for any permutation the
            // permute kernel writes); otherwise flag it and store nothing for this tile.
            const bool rows_ok = a.dense || ti.row0 + ti.n <= (ti.shared ? a.T : a.T * a.K);
            if (!rows_ok && lane == 0) set_dev_error(a.err, MOE_DEVERR_BAD_INDEX);
            const int f = ti.ft * BM + q * 32 + lane;
            const int feat = ti.shared ? a.feat_s : a.feat_r;
            const bool fok = f < feat;
            const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * C::kAccStride);
#pragma unroll
            for (int ci = 0; ci < kChunks; ++ci) {
                const int c0 = 32 * half + 32 * nhalf * ci;
                if (c0 >= ti.n || !rows_ok) break;
                uint32_t v[32];
                tmem_ld32(tb + c0, v);
                uint32_t u[32];
                if (C::kSwiglu) tmem_ld32(tb + C::kBN + c0, u);
                tmem_ld_wait();
                if (C::kGather) {
                    bf16* dst = ti.shared ? a.hs : a.h;
                    const int ld = feat;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int col = c0 + j;
                        if (col < ti.n && fok) {
                            float val;
                            if (C::kSwiglu) val = act_swiglu(__uint_as_float(v[j]), __uint_as_float(u[j]));
                            else val = act_relu2(__uint_as_float(v[j]));
                            dst[(size_t)(ti.row0 + col) * ld + f] = __float2bfloat16_rn(val);
                        }
                    }
                } else if (MODE == GM_FC2) {
                    if (ti.shared) {  // shared rows are the tokens in order; optional sigmoid gate
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int col = c0 + j;
                            if (col < ti.n && fok) {
                                float y = __uint_as_float(v[j]);
                                if (a.sgate) y = __fmul_rn(a.sgate[ti.row0 + col], y);
                                a.acc_s[(size_t)(ti.row0 + col) * a.feat_s + f] = y;
                            }
                        }
                    } else {
                        // Column j of this chunk is token t_j with routing weight w_j; lane l
                        // holds feature f0 + l.  Each block of 4 columns is transposed within
                        // groups of 4 lanes (two XOR-shuffle stages), after which lane 4g+i
                        // holds features f0+4g .. f0+4g+3 of token t_{j0+i}, scales them by
                        // w_{j0+i} (one shuffle brings the token, one the weight) and adds
                        // them into acc with one 16-byte vector reduction (FP32 add in L2).
                        // No shared memory is staged, so the ring keeps it for weights.
                        const int i4 = lane & 3;
                        const bool fok4 = f - i4 + 3 < a.feat_r;  // features of my group (feat_r % 8 == 0)
#pragma unroll
                        for (int j0 = 0; j0 < 32; j0 += 4) {
                            float r[4];
#pragma unroll
                            for (int jj = 0; jj < 4; ++jj) r[jj] = __uint_as_float(v[j0 + jj]);
                            // r[jj] = y[feature of this lane, token j0 + jj]; 4x4 transpose
                            float t0 = (i4 & 1) ? r[0] : r[1], t1 = (i4 & 1) ? r[2] : r[3];
                            t0 = __shfl_xor_sync(0xffffffffu, t0, 1);
                            t1 = __shfl_xor_sync(0xffffffffu, t1, 1);
                            if (i4 & 1) {
                                r[0] = t0;
                                r[2] = t1;
                            } else {
                                r[1] = t0;
                                r[3] = t1;
                            }
                            float u0 = (i4 & 2) ? r[0] : r[2], u1 = (i4 & 2) ? r[1] : r[3];
                            u0 = __shfl_xor_sync(0xffffffffu, u0, 2);
                            u1 = __shfl_xor_sync(0xffffffffu, u1, 2);
                            if (i4 & 2) {
                                r[0] = u0;
                                r[1] = u1;
                            } else {
                                r[2] = u0;
                                r[3] = u1;
                            }
                            const int tok = __shfl_sync(0xffffffffu, mt[ci], j0 + i4);
                            const float wt = __shfl_sync(0xffffffffu, mw[ci], j0 + i4);
                            if (c0 + j0 + i4 < ti.n && fok4 && (unsigned)tok < (unsigned)a.T)
                                red_add_v4_f32(a.acc + (size_t)tok * a.feat_r + (f - i4), wt * r[0], wt * r[1],
                                               wt * r[2], wt * r[3]);
                        }
                    }
                } else {  // GM_DENSE
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int col = c0 + j;
                        if (col < ti.n && fok) {
                            const float val = __uint_as_float(v[j]);
                            a.logits[(size_t)(ti.row0 + col) * a.feat_r + f] = val;
                            if (a.logits_copy) a.logits_copy[(size_t)(ti.row0 + col) * a.feat_r + f] = val;
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty_bar(buf));
        }
        if (trow && threadIdx.x == 64) trow[MOE_TRACE_STORES_DONE] = globaltimer_ns();
    } else if (C::kGather) {
        // ------------------------------------------------------------ FC1 token gather
        const int p = threadIdx.x - (64 + 32 * C::kEpiWarps);  // 0 .. kGatherThreads - 1
        const int chunk = p & 7, rsub = p >> 3;
        int it = 0;
        for (int tile = DYN ? id_consume(true) : (int)blockIdx.x; tile < total && !*abort_flag;
             tile = DYN ? id_consume(true) : tile + (int)gridDim.x) {
            const TileInfo ti = decode_tile<C::kBN>(a, s_tiles, s_offs, G, tile);
            const int kd = ti.shared ? a.kdim_s : a.kdim;
            const int nk = ti.nk;
            const int npad = cdiv(ti.n, 16) * 16;
            int tok[C::kBN / C::kGatherRowStep];
#pragma unroll
            for (int j = 0; j < C::kBN / C::kGatherRowStep; ++j) {
                const int r = rsub + C::kGatherRowStep * j;
                tok[j] = -1;
                if (r < ti.n && (ti.shared || ti.row0 + ti.n <= a.T * a.K)) {
                    const int src = ti.shared ? ti.row0 + r : a.perm[ti.row0 + r];
                    if ((unsigned)src < (unsigned)(ti.shared ? a.T : a.T * a.K)) {
                        tok[j] = ti.shared ? src : src % a.T;
                    } else {  // never from a valid permutation: flag it, gather zeros
                        set_dev_error(a.err, MOE_DEVERR_BAD_INDEX);
                    }
                }
            }
            bool ok = true;
            for (int kb = 0; kb < nk; ++kb, ++it) {
                const int s = it % C::kStages;
                const uint32_t ph = (uint32_t)(it / C::kStages) & 1u;
                if (!mbar_wait(empty_bar(s), ph ^ 1u, abort_flag, a.err)) {
                    ok = false;
                    break;
                }
                const uint32_t bs = base_u32 + (uint32_t)s * C::kStageBytes + C::kNA * A_BYTES;
                const int kcol = kb * BK + chunk * 8;
#pragma unroll
                for (int j = 0; j < C::kBN / C::kGatherRowStep; ++j) {
                    const int r = rsub + C::kGatherRowStep * j;
                    if (r < npad) {
                        const uint32_t dst = bs + (uint32_t)r * 128u + ((uint32_t)(chunk ^ (r & 7)) << 4);
                        const bool v = tok[j] >= 0 && kcol < kd;
                        const bf16* src = v ? a.xsrc + (size_t)tok[j] * a.kdim + kcol : a.xsrc;
                        cp_async16(dst, src, v ? 16u : 0u);
                    }
                }
                cp_async_commit();
                if (it >= C::kLag) {
                    cp_async_wait<C::kLag>();
                    fence_proxy_async_smem();
                    mbar_arrive(full_bar((it - C::kLag) % C::kStages));
                }
            }
            if (!ok) break;
        }
        cp_async_wait<0>();
        fence_proxy_async_smem();
        for (int j = max(0, it - C::kLag); j < it; ++j) mbar_arrive(full_bar(j % C::kStages));
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (*abort_flag) {  // let in-flight bulk copies and MMAs land before the CTA retires
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 50000ull) {
        }
    }
    if (trow && threadIdx.x == 0) trow[MOE_TRACE_EXIT] = globaltimer_ns();
    if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
    if (MODE == GM_DENSE) pdl_wait();  // the previous kernel is complete before this one is
    pdl_trigger();
}

// The stream-K kernel, launched for few-token calls (FC1 token tiles of 32 or 64 rows, FC2
// of 32 or 128): it decides on the device, from the call's tile count, between stream-K
// and whole tiles.  SK is always true here; it keeps the walker's whole-tile path compiled.
template <int MODE, int BN, bool SK>
__global__ void __launch_bounds__(Cfg<MODE, BN>::kThreads, 1)
    gemm_sk_kernel(const GemmArgs a, const __grid_constant__ CUtensorMap tm_a_r, const __grid_constant__ CUtensorMap tm_a_s,
                const __grid_constant__ CUtensorMap tm_b_r, const __grid_constant__ CUtensorMap tm_b_s) {
    using C = Cfg<MODE, BN>;
    // FC1's stream-K fix-up keeps [kNA][BN][128] partial sums per CTA: BN <= 64 only.
    constexpr bool kFix = SK && C::kGather && BN <= kStreamKMaxBN;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t base_u32 = (raw_u32 + 1023u) & ~1023u;
    uint8_t* base = smem_raw + (base_u32 - raw_u32);
    uint8_t* meta = base + (size_t)C::kStages * C::kStageBytes + C::kEpiBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(meta);  // full[S], empty[S], tfull[2], tempty[2]
    const uint32_t bar_u32 = smem_u32(bars);
    auto full_bar = [&](int s) { return bar_u32 + 8u * s; };
    auto empty_bar = [&](int s) { return bar_u32 + 8u * (C::kStages + s); };
    auto tfull_bar = [&](int b) { return bar_u32 + 8u * (2 * C::kStages + b); };
    auto tempty_bar = [&](int b) { return bar_u32 + 8u * (2 * C::kStages + 2 + b); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(meta + 8 * (2 * C::kStages + 4));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* s_tiles = reinterpret_cast<int*>(meta + 256);
    int* s_offs = s_tiles + C::kMaxGroups + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = a.E + (a.has_shared ? 1 : 0);
    // Phase trace (optional): this CTA's row of the kernel's trace block.
    unsigned long long* trow = a.trace ? a.trace + (size_t)blockIdx.x * MOE_TRACE_FIELDS : nullptr;
    if (trow && threadIdx.x == 0) trow[MOE_TRACE_ENTRY] = globaltimer_ns();

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(full_bar(s), 1 + C::kGatherThreads);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), C::kEpiWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_a_r);
        if (a.has_shared) tma_prefetch_desc(&tm_a_s);
        if (!C::kGather) {
            tma_prefetch_desc(&tm_b_r);
            if (a.has_shared) tma_prefetch_desc(&tm_b_s);
        }
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);

    // Everything below reads what earlier kernels wrote (tile tables, perm, h) -- except
    // in DENSE mode, which reads only the caller's x and Wr and waits at its end.
    if (MODE != GM_DENSE) pdl_wait();
    if (!a.dense) {
        for (int i = threadIdx.x; i <= G; i += blockDim.x) s_tiles[i] = a.tiles[i];
        for (int i = threadIdx.x; i <= a.E; i += blockDim.x) s_offs[i] = a.offsets[i];
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (trow && threadIdx.x == 0) trow[MOE_TRACE_READY] = globaltimer_ns();
    const uint32_t tmem_base = *tmem_slot;
    const int total = a.dense ? a.nfeat_r * cdiv(a.T, kDenseTokenTile) : s_tiles[G];
    const int routed_tiles = (a.dense || !a.has_shared) ? total : s_tiles[a.E];
    // Stream-K only where dealing whole tiles would leave the last wave mostly idle: more
    // tiles than CTAs, but under three quarters of the whole-tile waves' slots filled
    // (measured: with fewer tiles than SMs, or with several full waves, whole tiles are as
    // fast or faster).
    const int waves = cdiv(total, (int)gridDim.x);
    const bool streamk = SK && total > (int)gridDim.x && total < a.streamk_max &&
                         4 * total < 3 * waves * (int)gridDim.x;
    const int nk_r = cdiv(a.kdim, BK), nk_s = cdiv(a.kdim_s > 0 ? a.kdim_s : a.kdim, BK);
    // Round-robin dealing keeps the CTAs on neighbouring tiles of the group-major list (one
    // expert's feature and token tiles), which share that expert's weight and token rows in
    // L2, and spreads tiles of unequal cost (ragged token tails) evenly.
    WorkWalk<SK> work;
    work.init(total, routed_tiles, nk_r, nk_s, streamk);
    Seg sg;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t wpol = l2_policy_evict_first();
            int it = 0, units = 0;
            while (!*abort_flag && work.next(sg)) {
                const TileInfo ti = decode_tile<C::kBN>(a, s_tiles, s_offs, G, sg.tile);
                if (ti.nk == 0) continue;
                const bool sh = ti.shared;
                const CUtensorMap* ta = sh ? &tm_a_s : &tm_a_r;
                const CUtensorMap* tb = sh ? &tm_b_s : &tm_b_r;
                const int frow = ti.ft * BM;
                constexpr int BBOX = b_box_rows<MODE>();
                const int nbox = cdiv(ti.n, BBOX);
                const uint32_t bytes = C::kNA * A_BYTES + (C::kGather ? 0u : (uint32_t)nbox * BBOX * BK * 2);
                bool ok = true;
                for (int kb = sg.kb0; kb < sg.kb1; ++kb, ++it) {
                    const int s = it % C::kStages;
                    const uint32_t ph = (uint32_t)(it / C::kStages) & 1u;
                    if (!mbar_wait(empty_bar(s), ph ^ 1u, abort_flag, a.err)) {
                        ok = false;
                        break;
                    }
                    const uint32_t st = base_u32 + (uint32_t)s * C::kStageBytes;
                    mbar_expect_tx(full_bar(s), bytes);
                    if (sh || a.dense) {
                        tma_load_2d(st, ta, full_bar(s), kb * BK, frow);
                        if (C::kSwiglu) tma_load_2d(st + A_BYTES, ta, full_bar(s), kb * BK, a.up_s + frow);
                    } else if (MODE == GM_FC2 || ti.ntok == 1) {
                        // Weights that no other tile of this call reads: evict first, so that
                        // they do not push the token rows, h and the accumulator out of L2
                        // (measured on FC1: -9 % at 16 tokens, -6 % at 4096 tokens of the
                        // Qwen3.6-shaped layer).
                        tma_load_3d_hint(st, ta, full_bar(s), kb * BK, frow, ti.g, wpol);
                        if (C::kSwiglu)
                            tma_load_3d_hint(st + A_BYTES, ta, full_bar(s), kb * BK, a.up_r + frow, ti.g, wpol);
                    } else {  // a second token tile of this expert streams the same slice
                        tma_load_3d(st, ta, full_bar(s), kb * BK, frow, ti.g);
                        if (C::kSwiglu) tma_load_3d(st + A_BYTES, ta, full_bar(s), kb * BK, a.up_r + frow, ti.g);
                    }
                    if (!C::kGather) {
                        const uint32_t bs = st + C::kNA * A_BYTES;
                        for (int q = 0; q < nbox; ++q)
                            tma_load_2d(bs + (uint32_t)q * (BBOX * BK * 2), tb, full_bar(s), kb * BK,
                                        ti.row0 + q * BBOX);
                    }
                }
                if (!ok) break;
                ++units;
            }
            if (trow) {
                trow[MOE_TRACE_LOADS_DONE] = globaltimer_ns();
                trow[MOE_TRACE_UNITS] = (unsigned long long)units;
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int it = 0, tcount = 0;
            while (!*abort_flag && work.next(sg)) {
                const TileInfo ti = decode_tile<C::kBN>(a, s_tiles, s_offs, G, sg.tile);
                if (ti.nk == 0) continue;
                const int npad = cdiv(ti.n, 16) * 16;
                const uint32_t idesc = idesc_bf16_f32(BM, npad);
                const int buf = tcount % C::kAccBufs;
                const uint32_t tph = (uint32_t)(tcount / C::kAccBufs) & 1u;
                if (!mbar_wait(tempty_bar(buf), tph ^ 1u, abort_flag, a.err)) break;
                tc_fence_after();
                const uint32_t d0 = tmem_base + (uint32_t)(buf * C::kAccStride);
                const uint32_t d1 = d0 + C::kBN;
                bool ok = true;
                for (int kb = sg.kb0; kb < sg.kb1; ++kb, ++it) {
                    const int s = it % C::kStages;
                    const uint32_t ph = (uint32_t)(it / C::kStages) & 1u;
                    if (!mbar_wait(full_bar(s), ph, abort_flag, a.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = base_u32 + (uint32_t)s * C::kStageBytes;
                    const uint32_t bsm = st + C::kNA * A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint32_t accum = (kb > sg.kb0 || kk > 0) ? 1u : 0u;
                        const uint64_t bdesc = sdesc_sw128(bsm + kk * 32);
                        tc_mma(d0, sdesc_sw128(st + kk * 32), bdesc, idesc, accum);
                        if (C::kSwiglu) tc_mma(d1, sdesc_sw128(st + A_BYTES + kk * 32), bdesc, idesc, accum);
                    }
                    tc_commit(empty_bar(s));
                }
                if (!ok) break;
                tc_commit(tfull_bar(buf));
                ++tcount;
            }
        }
    } else if (warp < 2 + C::kEpiWarps) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                     // TMEM lane quarter of this warp
        const int half = (warp - 2) >> 2;          // which token columns (chunk parity)
        const int nhalf = C::kEpiWarps / 4;
        const int et = threadIdx.x - 64;
        if (a.zero_ptr) {
            float4* z = reinterpret_cast<float4*>(a.zero_ptr);
            const size_t n4 = a.zero_n / 4;
            const int ne = 32 * C::kEpiWarps;
            for (size_t i = (size_t)blockIdx.x * ne + et; i < n4; i += (size_t)gridDim.x * ne)
                z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        // FC1 stream-K scratch: one slot per CTA, [kNA][BN token columns][128 features] FP32.
        constexpr size_t kSlotFloats = (size_t)C::kNA * C::kBN * BM;
        int tcount = 0;
        // 32-token chunks per half of the epilogue warps (the last may lie past the tile)
        constexpr int kChunks = (C::kBN + 32 * (C::kEpiWarps / 4) - 1) / (32 * (C::kEpiWarps / 4));
        while (work.next(sg)) {
            const TileInfo ti = decode_tile<C::kBN>(a, s_tiles, s_offs, G, sg.tile);
            if (ti.nk == 0) continue;
            const int buf = tcount % C::kAccBufs;
            const uint32_t tph = (uint32_t)(tcount / C::kAccBufs) & 1u;
            // FC2: token and weight of each column this thread will scale, loaded before the
            // accumulator is ready (hidden behind the tile's mainloop).  Routed rows are
            // permuted slots (token, routing weight); the shared expert's rows are the tokens
            // in order (weight: the shared-expert gate, or 1).
            int mt[kChunks];
            float mw[kChunks];
#pragma unroll
            for (int ci = 0; ci < kChunks; ++ci) {
                mt[ci] = 0;
                mw[ci] = 0.0f;
                const int colm = 32 * half + 32 * nhalf * ci + lane;
                if (MODE == GM_FC2 && !ti.shared && colm < ti.n && ti.row0 + ti.n <= a.T * a.K) {
                    const int src = ld_nc_pinned_s32(a.perm + ti.row0 + colm);
                    if ((unsigned)src < (unsigned)(a.T * a.K)) {
                        const int kk = src / a.T;
                        mt[ci] = src - kk * a.T;
                        mw[ci] = ld_nc_pinned_f32(a.topk_w + (size_t)mt[ci] * a.K + kk);
                    } else {  // never from a valid permutation: flag it, contribute nothing
                        set_dev_error(a.err, MOE_DEVERR_BAD_INDEX);
                    }
                } else if (MODE == GM_FC2 && ti.shared && colm < ti.n) {
                    mt[ci] = ti.row0 + colm;
                    mw[ci] = a.sgate ? ld_nc_pinned_f32(a.sgate + mt[ci]) : 1.0f;
                }
            }
            const bool waited = mbar_wait(tfull_bar(buf), tph, abort_flag, a.err);
            if (!waited) break;
            tc_fence_after();
            // The tile's rows must lie inside their buffer (they do for any permutation the
            // permute kernel writes); otherwise flag it and store nothing for this tile.
            const bool rows_ok = a.dense || ti.row0 + ti.n <= (ti.shared ? a.T : a.T * a.K);
            if (!rows_ok && lane == 0) set_dev_error(a.err, MOE_DEVERR_BAD_INDEX);
            const int f = ti.ft * BM + q * 32 + lane;
            const int feat = ti.shared ? a.feat_s : a.feat_r;
            const bool fok = f < feat;
            const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * C::kAccStride);
            if (kFix && sg.kind == kPart) {
                // ---- stream-K, FC1: a later k-block range; its partial sums go to this CTA's
                // slot, then the tile's counter tells the fixer it is there.
                float* slot = a.skp + (size_t)blockIdx.x * kSlotFloats;
#pragma unroll
                for (int ci = 0; ci < kChunks; ++ci) {
                    const int c0 = 32 * half + 32 * nhalf * ci;
                    if (c0 >= ti.n || !rows_ok) break;
                    uint32_t v[32];
                    tmem_ld32(tb + c0, v);
                    uint32_t u[32];
                    if (C::kSwiglu) tmem_ld32(tb + C::kBN + c0, u);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int col = c0 + j;
                        if (col < ti.n) {
                            slot[(size_t)col * BM + q * 32 + lane] = __uint_as_float(v[j]);
                            if (C::kSwiglu) slot[(size_t)(C::kBN + col) * BM + q * 32 + lane] = __uint_as_float(u[j]);
                        }
                    }
                }
                // Each warp publishes its own rows: every lane's stores are fenced, then the
                // warp's lane 0 counts it on the tile's counter (no barrier across warps).
                __threadfence();
                __syncwarp();
                if (lane == 0) atomicAdd(a.done + sg.tile, 1);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(tempty_bar(buf));
                ++tcount;
                continue;
            }
            int ncontrib = 0;
            if (kFix && sg.kind == kFixer) {
                // ---- stream-K, FC1: this CTA holds the tile's first k-blocks.  Each warp waits
                // (bounded) until every warp of every later range has published its partial,
                // then adds them below.
                for (int c = blockIdx.x + 1; c <= sg.last; ++c) ncontrib += work.active(c) ? 1 : 0;
                int ok = 1;
                if (lane == 0) {
                    const volatile int* cnt = a.done + sg.tile;
                    const int target = ncontrib * C::kEpiWarps;
                    const uint64_t t0 = globaltimer_ns();
                    uint32_t n = 0;
                    while (*cnt < target) {
                        if ((++n & 255u) == 0) {
                            if (*abort_flag) {
                                ok = 0;
                                break;
                            }
                            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                                *abort_flag = 1;
                                set_dev_error(a.err, MOE_DEVERR_WAIT_TIMEOUT);
                                ok = 0;
                                break;
                            }
                        }
                    }
                    __threadfence();
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
            }
#pragma unroll
            for (int ci = 0; ci < kChunks; ++ci) {
                const int c0 = 32 * half + 32 * nhalf * ci;
                if (c0 >= ti.n || !rows_ok) break;
                uint32_t v[32];
                tmem_ld32(tb + c0, v);
                uint32_t u[32];
                if (C::kSwiglu) tmem_ld32(tb + C::kBN + c0, u);
                tmem_ld_wait();
                if (kFix && ncontrib > 0) {  // the later ranges' partial sums, in CTA order
                    for (int c = blockIdx.x + 1; c <= sg.last; ++c) {
                        if (!work.active(c)) continue;
                        const float* slot = a.skp + (size_t)c * kSlotFloats;
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int col = c0 + j;
                            if (col < ti.n) {
                                v[j] = __float_as_uint(__uint_as_float(v[j]) +
                                                       __ldcg(slot + (size_t)col * BM + q * 32 + lane));
                                if (C::kSwiglu)
                                    u[j] = __float_as_uint(__uint_as_float(u[j]) +
                                                           __ldcg(slot + (size_t)(C::kBN + col) * BM + q * 32 + lane));
                            }
                        }
                    }
                }
                if (C::kGather) {
                    bf16* dst = ti.shared ? a.hs : a.h;
                    const int ld = feat;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int col = c0 + j;
                        if (col < ti.n && fok) {
                            float val;
                            if (C::kSwiglu) val = act_swiglu(__uint_as_float(v[j]), __uint_as_float(u[j]));
                            else val = act_relu2(__uint_as_float(v[j]));
                            dst[(size_t)(ti.row0 + col) * ld + f] = __float2bfloat16_rn(val);
                        }
                    }
                } else if (MODE == GM_FC2) {
                    // Column j of this chunk is token t_j with weight w_j; lane l holds feature
                    // f0 + l.  Each block of 4 columns is transposed within groups of 4 lanes
                    // (two XOR-shuffle stages), after which lane 4g+i holds features
                    // f0+4g .. f0+4g+3 of token t_{j0+i}, scales them by w_{j0+i} (one shuffle
                    // brings the token, one the weight) and adds them into the FP32
                    // accumulator (routed rows: acc; the shared expert: acc_s) with one 16-byte
                    // vector reduction (FP32 add in L2).  A stream-K range adds its partial
                    // sum the same way.  No shared memory is staged, so the ring keeps it for
                    // weights.
                    if (ti.shared) combine_chunk(v, mt[ci], mw[ci], c0, ti.n, f, a.feat_s, a.T, a.acc_s, lane);
                    else combine_chunk(v, mt[ci], mw[ci], c0, ti.n, f, a.feat_r, a.T, a.acc, lane);
                } else {  // GM_DENSE
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int col = c0 + j;
                        if (col < ti.n && fok) {
                            const float val = __uint_as_float(v[j]);
                            a.logits[(size_t)(ti.row0 + col) * a.feat_r + f] = val;
                            if (a.logits_copy) a.logits_copy[(size_t)(ti.row0 + col) * a.feat_r + f] = val;
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty_bar(buf));
            ++tcount;
        }
        if (trow && threadIdx.x == 64) trow[MOE_TRACE_STORES_DONE] = globaltimer_ns();
    } else if (C::kGather) {
        // ------------------------------------------------------------ FC1 token gather
        const int p = threadIdx.x - (64 + 32 * C::kEpiWarps);  // 0 .. kGatherThreads - 1
        const int chunk = p & 7, rsub = p >> 3;
        int it = 0;
        while (!*abort_flag && work.next(sg)) {
            const TileInfo ti = decode_tile<C::kBN>(a, s_tiles, s_offs, G, sg.tile);
            if (ti.nk == 0) continue;
            const int kd = ti.shared ? a.kdim_s : a.kdim;
            const int npad = cdiv(ti.n, 16) * 16;
            int tok[C::kBN / C::kGatherRowStep];
#pragma unroll
            for (int j = 0; j < C::kBN / C::kGatherRowStep; ++j) {
                const int r = rsub + C::kGatherRowStep * j;
                tok[j] = -1;
                if (r < ti.n && (ti.shared || ti.row0 + ti.n <= a.T * a.K)) {
                    const int src = ti.shared ? ti.row0 + r : a.perm[ti.row0 + r];
                    if ((unsigned)src < (unsigned)(ti.shared ? a.T : a.T * a.K)) {
                        tok[j] = ti.shared ? src : src % a.T;
                    } else {  // never from a valid permutation: flag it, gather zeros
                        set_dev_error(a.err, MOE_DEVERR_BAD_INDEX);
                    }
                }
            }
            bool ok = true;
            for (int kb = sg.kb0; kb < sg.kb1; ++kb, ++it) {
                const int s = it % C::kStages;
                const uint32_t ph = (uint32_t)(it / C::kStages) & 1u;
                if (!mbar_wait(empty_bar(s), ph ^ 1u, abort_flag, a.err)) {
                    ok = false;
                    break;
                }
                const uint32_t bs = base_u32 + (uint32_t)s * C::kStageBytes + C::kNA * A_BYTES;
                const int kcol = kb * BK + chunk * 8;
#pragma unroll
                for (int j = 0; j < C::kBN / C::kGatherRowStep; ++j) {
                    const int r = rsub + C::kGatherRowStep * j;
                    if (r < npad) {
                        const uint32_t dst = bs + (uint32_t)r * 128u + ((uint32_t)(chunk ^ (r & 7)) << 4);
                        const bool v = tok[j] >= 0 && kcol < kd;
                        const bf16* src = v ? a.xsrc + (size_t)tok[j] * a.kdim + kcol : a.xsrc;
                        cp_async16(dst, src, v ? 16u : 0u);
                    }
                }
                cp_async_commit();
                if (it >= C::kLag) {
                    cp_async_wait<C::kLag>();
                    fence_proxy_async_smem();
                    mbar_arrive(full_bar((it - C::kLag) % C::kStages));
                }
            }
            if (!ok) break;
        }
        cp_async_wait<0>();
        fence_proxy_async_smem();
        for (int j = max(0, it - C::kLag); j < it; ++j) mbar_arrive(full_bar(j % C::kStages));
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (*abort_flag) {  // let in-flight bulk copies and MMAs land before the CTA retires
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 50000ull) {
        }
    }
    if (trow && threadIdx.x == 0) trow[MOE_TRACE_EXIT] = globaltimer_ns();
    if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
    if (MODE == GM_DENSE) pdl_wait();  // the previous kernel is complete before this one is
    pdl_trigger();
}

// ---------------------------------------------------------------- finalize
// `sh_out` may be the caller's shared output and `out` that same buffer: each thread reads
// its 8 elements before writing them, so the in-place form is safe (no __restrict__).
__global__ void __launch_bounds__(256) finalize_kernel(const float* __restrict__ acc, const float* __restrict__ acc_s,
                                                       const bf16* sh_out, bf16* out, size_t n, float scale) {
    pdl_wait();
    const size_t stride = (size_t)gridDim.x * blockDim.x * 8;
    for (size_t i = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) * 8; i < n; i += stride) {
        const float4 a0 = *reinterpret_cast<const float4*>(acc + i);
        const float4 a1 = *reinterpret_cast<const float4*>(acc + i + 4);
        float r[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        if (scale != 1.0f) {
#pragma unroll
            for (int j = 0; j < 8; ++j) r[j] = __fmul_rn(scale, r[j]);
        }
        if (acc_s) {  // routed -> BF16, shared -> BF16, BF16 add
            const float4 s0 = *reinterpret_cast<const float4*>(acc_s + i);
            const float4 s1 = *reinterpret_cast<const float4*>(acc_s + i + 4);
            const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
            for (int j = 0; j < 8; ++j) r[j] = __fadd_rn(bf_round(r[j]), bf_round(sv[j]));
        } else if (sh_out) {
            const uint4 y = *reinterpret_cast<const uint4*>(sh_out + i);
            const uint32_t yw[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                r[2 * j] = __fadd_rn(bf_round(r[2 * j]), bf16lo(yw[j]));
                r[2 * j + 1] = __fadd_rn(bf_round(r[2 * j + 1]), bf16hi(yw[j]));
            }
        }
        uint4 o;
        o.x = (uint32_t)f2bf_bits(r[0]) | ((uint32_t)f2bf_bits(r[1]) << 16);
        o.y = (uint32_t)f2bf_bits(r[2]) | ((uint32_t)f2bf_bits(r[3]) << 16);
        o.z = (uint32_t)f2bf_bits(r[4]) | ((uint32_t)f2bf_bits(r[5]) << 16);
        o.w = (uint32_t)f2bf_bits(r[6]) | ((uint32_t)f2bf_bits(r[7]) << 16);
        *reinterpret_cast<uint4*>(out + i) = o;
    }
    pdl_trigger();
}

}  // namespace

template <typename Kern>
static cudaError_t launch_gemm_kernel(Kern kern, size_t smem, int threads, const GemmArgs& a, const GemmMaps& m,
                                      int grid, cudaStream_t s, bool pdl) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_k(kern, dim3(grid), dim3(threads), smem, s, pdl, a, m.a_r, m.a_s, m.b_r, m.b_s);
}
// The stream-K kernel exists for the token tiles of few-token calls (32 and 64 rows for
// FC1, 32 and 128 for FC2); a.streamk_max == 0 selects the whole-tile kernel.
template <int MODE, int BN>
static cudaError_t launch_mode(const GemmArgs& a, const GemmMaps& m, int grid, cudaStream_t s, bool pdl) {
    using C = Cfg<MODE, BN>;
    constexpr bool kHasSK = MODE == GM_FC2 ? (BN == 32 || BN == 128) : (MODE != GM_DENSE && BN <= kStreamKMaxBN);
    if constexpr (kHasSK) {
        if (a.streamk_max > 0)
            return launch_gemm_kernel(gemm_sk_kernel<MODE, BN, true>, C::kSmem, C::kThreads, a, m, grid, s, pdl);
    }
    if constexpr (MODE != GM_DENSE) {
        if (a.dyn_ctr) return launch_gemm_kernel(gemm_kernel<MODE, BN, true>, C::kSmem, C::kThreads, a, m, grid, s, pdl);
    }
    return launch_gemm_kernel(gemm_kernel<MODE, BN, false>, C::kSmem, C::kThreads, a, m, grid, s, pdl);
}

int gemm_token_tile(int mode, int T, int K, int E) {
    if (mode == GM_DENSE) return kDenseTokenTile;
    if (T <= 32) return 32;  // no expert has more rows than a tile
    const double rows = (double)T * K / E;  // average rows per expert
    // FC2: a tile that covers an expert's rows streams its W2 slice once; 192 holds almost
    // every expert of ~128 rows with 5 stages (measured: 160 with 6 stages is no faster).
    if (mode == GM_FC2) return rows <= 64.0 ? 128 : (rows <= 150.0 ? 192 : 256);
    // FC1: a tile re-streams the expert's weight slice, so an expert just over a tile's
    // width costs a second, nearly empty tile; 256-token tiles keep most experts at one.
    // Not for SwiGLU: its 256-token stage (64 KB) leaves room for only 3 stages, and the
    // bytes in flight per SM, not the tile count, set the time (measured: 128 is ahead at
    // 128 and 256 rows per expert).  Nor a 160-token SwiGLU tile whose gate and up take
    // both TMEM buffers when it holds more than 128 rows: it serialises those tiles'
    // epilogues with the mainloops around them (measured 1.5x slower at 256 rows).
    if (mode == GM_FC1_SWIGLU) return rows <= 48.0 ? 64 : 128;
    return rows <= 48.0 ? 64 : (rows <= 96.0 ? 128 : 256);
}

cudaError_t launch_gemm(int mode, int bn, const GemmArgs& a, const GemmMaps& m, int grid, cudaStream_t s, bool pdl) {
    switch (mode) {
        case GM_FC1_SWIGLU:
            if (bn == 32) return launch_mode<GM_FC1_SWIGLU, 32>(a, m, grid, s, pdl);
            if (bn == 64) return launch_mode<GM_FC1_SWIGLU, 64>(a, m, grid, s, pdl);
            if (bn == 128) return launch_mode<GM_FC1_SWIGLU, 128>(a, m, grid, s, pdl);
            break;
        case GM_FC1_RELU2:
            if (bn == 32) return launch_mode<GM_FC1_RELU2, 32>(a, m, grid, s, pdl);
            if (bn == 64) return launch_mode<GM_FC1_RELU2, 64>(a, m, grid, s, pdl);
            if (bn == 128) return launch_mode<GM_FC1_RELU2, 128>(a, m, grid, s, pdl);
            if (bn == 256) return launch_mode<GM_FC1_RELU2, 256>(a, m, grid, s, pdl);
            break;
        case GM_FC2:
            if (bn == 32) return launch_mode<GM_FC2, 32>(a, m, grid, s, pdl);
            if (bn == 128) return launch_mode<GM_FC2, 128>(a, m, grid, s, pdl);
            if (bn == 192) return launch_mode<GM_FC2, 192>(a, m, grid, s, pdl);
            if (bn == 256) return launch_mode<GM_FC2, 256>(a, m, grid, s, pdl);
            break;
        case GM_DENSE: return launch_mode<GM_DENSE, kDenseTokenTile>(a, m, grid, s, pdl);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_finalize(const float* acc, const float* acc_s, const bf16* sh_out, bf16* out, size_t n,
                            float scale, int num_sms, cudaStream_t s, bool pdl) {
    const size_t groups = n / 8;
    int grid = (int)std::min<size_t>((groups + 255) / 256, (size_t)num_sms * 4);
    if (grid < 1) grid = 1;
    return launch_k(finalize_kernel, dim3(grid), dim3(256), 0, s, pdl, acc, acc_s, sh_out, out, n, scale);
}

size_t fc1_streamk_bytes(int bn, bool swiglu, int grid) {
    if (bn > kStreamKMaxBN) return 0;
    return (size_t)grid * (swiglu ? 2 : 1) * bn * BM * sizeof(float);
}

int gemm_streamk_max(int mode, int bn, int grid, long long max_tiles) {
    if (mode == GM_DENSE) return 0;
    if (mode == GM_FC2) {
        if (bn != 32 && bn != 128) return 0;
    } else if (bn > kStreamKMaxBN) {
        return 0;
    }
    const int limit = mode == GM_FC2 ? kStreamKWaves * grid : std::min(kStreamKWaves * grid, kStreamKMaxTiles);
    return max_tiles < limit ? limit : 0;  // the call can have fewer tiles than the limit
}

}  // namespace moe
