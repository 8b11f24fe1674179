// fused_decode_sm100.cu -- the whole MoE layer for a decode batch (bf16
// weights) in one persistent kernel: routing, bucketing, the gate/up grouped
// GEMM with SwiGLU, the down grouped GEMM and the weighted finalize.
//
// The steps are the layer's (InfiniLM PR #500 Qwen3-MoE report §2.1-§2.2;
// FlashInfer PR #7196 analysis §1 for finalize, §2 for the runtime-N tiles;
// the GC-MoE abstract fuses the layer's steps into one graph). One launch, no
// host synchronisation and no kernel boundary between the steps:
//  - Before it waits for the previous kernel, every CTA prefetches into L2 the
//    first K-blocks of the gate/up weights of the CTA-th tile, so HBM streams
//    weights while the batch is routed (weights are constant inputs).
//  - CTA t < T routes token t (route_token, one warp) into the workspace and
//    counts it (release); every CTA waits for the T tokens (acquire, bounded)
//    and buckets the whole batch in shared memory from per-expert token
//    masks (bit t of mask[e]: token t has a slot routed to e). A token has at
//    most one slot per expert, so the rank of slot (t, j) inside expert e is
//    the number of lower tokens in mask[e]: the stable order by slot id that
//    the permute kernels produce, with no histogram passes.
//  - Tiles: 256 weight rows (two M = 128 halves sharing the token operand) x
//    all tokens of one expert (N = align16(count) <= 64). Gate/up tile of
//    expert e and 128-feature block mb: half 0 = gate rows, half 1 = up rows;
//    down tile: halves = output rows mb*256 .. +127 and +128 .. +255. Both
//    kinds have the same shared-memory stage (32 KB of weights + 8 KB of
//    token rows, K = 64) and the same TMEM accumulators.
//  - The tile list (gate/up tiles of the non-empty experts, then their down
//    tiles) is handed out dynamically: the producer warp takes the next tile
//    number from a counter in global memory and passes it to the MMA and
//    epilogue warps through a queue in shared memory. A CTA holds no tile it
//    has not started, so no CTA waits on a CTA that is not running, and the
//    CTAs finish together whatever the tiles' sizes.
//  - A down tile of expert e reads act rows written by the gate/up tiles of
//    e, which may run on other CTAs: their epilogues count finished tiles per
//    expert in global memory (release). The producer loads the down tile's
//    first weight stages, then waits for the count (acquire, bounded), then
//    loads act. Finalize waits likewise for the count of finished down
//    tiles; then every CTA combines a share of the tokens in the finalize
//    kernel's order of operations.
//  - A one-warp reset kernel zeroes the counters before each call; both are
//    launched with programmatic dependent launch, so the reset and this
//    kernel's set-up and prefetch overlap the previous kernel's tail.
#include "gemm_common.cuh"
#include "launch_util.cuh"
#include "route_dev.cuh"

namespace moe {
namespace {

using namespace gemm;

constexpr int kFThreads = 256;          // 0 TMA, 1 MMA, 2-5 epilogue; all 8 warps route, bucket and finalize
constexpr int kFWarps = kFThreads / 32;
constexpr int kFBN = 64;                // token rows per tile: every token of one expert (T <= 64)
constexpr int kFMaxT = 64;
constexpr int kFMaxSlots = 16;
constexpr int kFMaxP = kFMaxT * kFMaxSlots;
constexpr int kFMaxE = 256;
constexpr int kFStages = 5;
constexpr int kFBBytes = kFBN * kBK * 2;                    // 8 KB of token rows per stage
constexpr int kFSlot = 2 * kTileBytesA + kFBBytes;          // 40 KB: two weight halves + token rows (K = 64)
constexpr int kFAccCols = 2 * kFBN;                         // per TMEM buffer: half 0, half 1
constexpr int kFTmemCols = 2 * kFAccCols;
constexpr int kFQueue = 8;                                  // tile numbers in flight between the roles
constexpr int kFPrefetchKB = 6;                             // K-blocks prefetched to L2 before routing
constexpr unsigned long long kFDepLimitNs = 2000000000ull;

struct FusedArgs {
    const float *logits;
    int T, E, k, S, H, I;               // E routed experts, k routed slots, S shared experts
    int32_t *ids, *counts, *offsets, *perm, *inv_perm;   // workspace copies of the routing / permutation
    float *w;
    uint16_t *act;                      // [P, I]
    uint16_t *y;                        // [P, H]
    uint16_t *out;                      // [T, H]
    unsigned int *gu_done;              // [E + S] finished gate/up tiles x 4 epilogue warps, per expert
    unsigned int *dn_done;              // [1] finished down tiles x 4 epilogue warps
    unsigned int *next_tile;            // [1] tiles handed out
    unsigned int *routed;               // [1] tokens routed
    int *err;
};

struct FusedSmem {
    unsigned long long mask[kFMaxE];    // bit t: token t has a slot routed to expert e
    int32_t ids[kFMaxP];
    int32_t perm[kFMaxP];
    int32_t inv[kFMaxP];
    float w[kFMaxP];
    int off[kFMaxE + 1];
    int ne[kFMaxE];                     // non-empty experts, ascending
    int n_ne;
    int first_tile;
    int warp_sums[kFWarps];
    int tile_q[kFQueue];
};

__device__ __forceinline__ unsigned int ld_acquire_u32(const unsigned int *p) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void red_release_add_u32(unsigned int *p, unsigned int v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Generic-proxy writes to global memory made visible to later async-proxy
// (TMA) reads.
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Waits until *p >= target (acquire), for at most kFDepLimitNs; false on a
// timeout (raises kErrTimeout and sets *abort) or when *abort is set.
__device__ bool wait_count(const unsigned int *p, unsigned int target, volatile int *abort, int *err) {
    if (ld_acquire_u32(p) >= target) return true;
    const unsigned long long t0 = globaltimer_ns();
    uint32_t sleep_ns = 32;
    while (ld_acquire_u32(p) < target) {
        if (*abort) return false;
        if (globaltimer_ns() - t0 > kFDepLimitNs) {
            raise_error(err, kErrTimeout);
            *abort = 1;
            return false;
        }
        __nanosleep(sleep_ns);
        if (sleep_ns < 512) sleep_ns <<= 1;
    }
    return true;
}

struct FTile {
    bool gu;        // gate/up tile (else down)
    bool two;       // a second 128-row half (always for gate/up)
    int h0;         // down: first 128-row half of the 256-row block (1 for the upper half of a split tile)
    int e, mb, row0, valid, n_mma;
};

// Tile numbers: [0, n_gu) gate/up tiles, expert-major; then the down tiles,
// expert-major, of which the last n_split (one per CTA) are split into their
// two 128-row halves, so that the tiles handed out last are the shortest.
struct TileCounts {
    int n_gu, n_dn, n_split;
    __device__ __forceinline__ int total() const { return n_gu + n_dn + n_split; }
};

__device__ __forceinline__ TileCounts tile_counts(const FusedSmem &fs, int MB_gu, int MB_dn) {
    TileCounts c;
    c.n_gu = fs.n_ne * MB_gu;
    c.n_dn = fs.n_ne * MB_dn;
    c.n_split = min(c.n_dn, static_cast<int>(gridDim.x));
    return c;
}

__device__ __forceinline__ FTile fused_tile(int tile, const TileCounts &c, const FusedSmem &fs, int MB_gu,
                                            int MB_dn, int H) {
    FTile f;
    f.gu = tile < c.n_gu;
    int local = f.gu ? tile : tile - c.n_gu;
    f.h0 = 0;
    bool split = false;
    if (!f.gu && local >= c.n_dn - c.n_split) {
        const int h = local - (c.n_dn - c.n_split);
        local = c.n_dn - c.n_split + h / 2;
        f.h0 = h & 1;
        split = true;
    }
    const int MB = f.gu ? MB_gu : MB_dn;
    f.e = fs.ne[local / MB];
    f.mb = local % MB;
    f.row0 = fs.off[f.e];
    f.valid = fs.off[f.e + 1] - f.row0;
    f.n_mma = (f.valid + 15) & ~15;
    f.two = f.gu || (!split && f.mb * 2 * kBM + kBM < H);
    return f;
}

// Queue entry qs: waits until it is filled, reads the tile number and frees
// the entry (one thread per consuming warp).
__device__ __forceinline__ bool pop_tile(const FusedSmem &fs, uint64_t *q_full, uint64_t *q_empty, int qs,
                                         uint32_t qph, volatile int *abort, int *err, int &tile) {
    if (!mbar_wait(&q_full[qs], qph, abort, err, 256)) return false;
    tile = reinterpret_cast<const volatile int *>(fs.tile_q)[qs];
    mbar_arrive(&q_empty[qs]);
    return true;
}

__global__ void __launch_bounds__(32) fused_reset_kernel(unsigned int *counters, int n) {
    griddep_launch_dependents();
    griddep_wait();                     // the previous call may still read its counters
    for (int i = threadIdx.x; i < n; i += 32) counters[i] = 0u;
}

template <int PER_LANE>
__global__ void __launch_bounds__(kFThreads, 1)
fused_decode_kernel(const __grid_constant__ CUtensorMap tmWgu, const __grid_constant__ CUtensorMap tmWd,
                    const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmAct,
                    const FusedArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *ring = smem;                                        // kFStages x kFSlot
    uint64_t *bars = reinterpret_cast<uint64_t *>(ring + kFStages * kFSlot);
    uint64_t *full_bar = bars;
    uint64_t *empty_bar = full_bar + kFStages;
    uint64_t *tfull_bar = empty_bar + kFStages;
    uint64_t *tempty_bar = tfull_bar + 2;
    uint64_t *q_full = tempty_bar + 2;
    uint64_t *q_empty = q_full + kFQueue;
    uint64_t *drain_bar = q_empty + kFQueue;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain_bar + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
    FusedSmem &fs = *reinterpret_cast<FusedSmem *>(tmem_holder + 16);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int K = a.k + a.S, Et = a.E + a.S, P = a.T * K;
    const int MB_gu = (a.I + kBM - 1) / kBM, MB_dn = (a.H + 2 * kBM - 1) / (2 * kBM);
    const int KB_gu = (a.H + kBK - 1) / kBK, KB_dn = (a.I + kBK - 1) / kBK;

    // ---- set-up and L2 prefetch (reads nothing written by earlier kernels) ----
    if (threadIdx.x == 0) {
        for (int s = 0; s < kFStages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull_bar[b], 1);
            mbar_init(&tempty_bar[b], kEpiThreads);
        }
        for (int q = 0; q < kFQueue; ++q) {
            mbar_init(&q_full[q], 1);
            mbar_init(&q_empty[q], 1 + kEpiThreads / 32);      // the MMA thread and one lane per epilogue warp
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmWgu);
        prefetch_tmap(&tmWd);
        prefetch_tmap(&tmX);
        prefetch_tmap(&tmAct);
        // the gate/up tile that this CTA's number names when no expert is
        // empty: the first tiles handed out are these, in some order
        const int e = blockIdx.x / MB_gu, mb = blockIdx.x % MB_gu;
        if (e < Et) {
            const int row = e * 2 * a.I + mb * kBM;
            for (int kb = 0; kb < kFPrefetchKB && kb < KB_gu; ++kb) {
                tma_prefetch_l2_2d(&tmWgu, kb * kBK, row);
                tma_prefetch_l2_2d(&tmWgu, kb * kBK, row + a.I);
            }
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, kFTmemCols);
        tmem_relinquish();
    }
    for (int e = threadIdx.x; e < kFMaxE; e += kFThreads) fs.mask[e] = 0ull;
    griddep_wait();
    // the first tile number: its round trip overlaps the routing
    unsigned int first_tile = 0;
    if (threadIdx.x == 0) first_tile = atomicAdd(a.next_tile, 1u);
    __syncthreads();

    // ---- routing: CTA t routes token t; every CTA reads the T tokens' slots ----
    if (warp == 0 && static_cast<int>(blockIdx.x) < a.T) {
        const int t = blockIdx.x;
        int id;
        float wt;
        route_token<PER_LANE>(a.logits + static_cast<size_t>(t) * a.E, a.E, a.k, id, wt);
        shared_slot(lane, a.k, a.E, id, wt);
        if (lane < K) {
            a.ids[t * K + lane] = id;
            a.w[t * K + lane] = wt;
        }
        __syncwarp();
        if (lane == 0) red_release_add_u32(a.routed, 1u);
    }
    if (threadIdx.x == 0) {
        fs.first_tile = static_cast<int>(first_tile);
        wait_count(a.routed, static_cast<unsigned int>(a.T), abort_flag, a.err);
    }
    __syncthreads();
    for (int s = threadIdx.x; s < P; s += kFThreads) {
        const int id = __ldcg(a.ids + s);
        const int t = s / K;
        fs.ids[s] = id;
        fs.w[s] = __ldcg(a.w + s);
        if (id >= 0 && id < Et) atomicOr(reinterpret_cast<unsigned int *>(&fs.mask[id]) + (t >> 5), 1u << (t & 31));
        else raise_error(a.err, kErrBadExpertId);
    }
    __syncthreads();
    // ---- bucketing: counts, offsets and the non-empty experts in one scan ------
    {
        const int e = threadIdx.x;                          // Et <= kFThreads
        const int c = e < Et ? __popcll(fs.mask[e]) : 0;
        const int packed = c | ((c > 0 ? 1 : 0) << 16);     // count (<= 1024) | non-empty flag
        int x = packed;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) fs.warp_sums[warp] = x;
        __syncthreads();
        int before = 0;
        for (int w = 0; w < warp; ++w) before += fs.warp_sums[w];
        const int excl = before + x - packed;
        if (e < Et) {
            fs.off[e] = excl & 0xFFFF;
            if (c > 0) fs.ne[excl >> 16] = e;
        }
        if (e == Et - 1) {
            fs.off[Et] = (excl + packed) & 0xFFFF;
            fs.n_ne = (excl + packed) >> 16;
        }
    }
    __syncthreads();
    for (int s = threadIdx.x; s < P; s += kFThreads) {
        const int t = s / K, e = min(max(fs.ids[s], 0), Et - 1);
        const int r = fs.off[e] + __popcll(fs.mask[e] & ((1ull << t) - 1ull));
        fs.perm[r] = s;
        fs.inv[s] = r;
    }
    __syncthreads();
    if (blockIdx.x == 0) {
        for (int i = threadIdx.x; i < P; i += kFThreads) {
            a.perm[i] = fs.perm[i];
            a.inv_perm[i] = fs.inv[i];
        }
        for (int e = threadIdx.x; e <= Et; e += kFThreads) {
            a.offsets[e] = fs.off[e];
            if (e < Et) a.counts[e] = fs.off[e + 1] - fs.off[e];
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_holder;
    const TileCounts tc = tile_counts(fs, MB_gu, MB_dn);
    const int total_tiles = tc.total();
    // token row of permuted row r (rows past P read row 0; they are never stored)
    auto token_of = [&](int r) { return r < P ? fs.perm[r] / K : 0; };

    if (warp == 0) {
        // ================================ TMA producer ==========================
        const uint64_t pol_w = l2_policy_evict_first();
        const uint64_t pol_x = l2_policy_evict_last();
        int stage = 0, qs = 0;
        uint32_t phase = 0, qph = 0;
        bool ok = true;
        int tile = fs.first_tile;
        while (ok) {
            const bool last = tile >= total_tiles;
            if (lane == 0) ok = mbar_wait(&q_empty[qs], qph ^ 1, abort_flag, a.err, 256);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            if (lane == 0) {
                reinterpret_cast<volatile int *>(fs.tile_q)[qs] = last ? -1 : tile;
                mbar_arrive(&q_full[qs]);
            }
            if (++qs == kFQueue) { qs = 0; qph ^= 1; }
            if (last) break;
            unsigned int next = 0;
            if (lane == 0) next = atomicAdd(a.next_tile, 1u);
            const FTile ft = fused_tile(tile, tc, fs, MB_gu, MB_dn, a.H);
            const int nbox = ft.n_mma / kBoxN;
            if (ft.gu) {
                const int row = ft.e * 2 * a.I + ft.mb * kBM;
                const uint32_t tx = 2 * kTileBytesA + nbox * kBoxBytesB;
                const bool gather_lane = 4 * lane < ft.n_mma;
                int tr[4] = {0, 0, 0, 0};
                if (gather_lane) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) tr[j] = token_of(ft.row0 + 4 * lane + j);
                }
                for (int kb = 0; kb < KB_gu; ++kb) {
                    if (lane == 0) ok = mbar_wait(&empty_bar[stage], phase ^ 1, abort_flag, a.err, 0);
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    uint8_t *st = ring + stage * kFSlot;
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&full_bar[stage], tx);
                        tma_load_2d(st, &tmWgu, &full_bar[stage], kb * kBK, row, pol_w);
                        tma_load_2d(st + kTileBytesA, &tmWgu, &full_bar[stage], kb * kBK, row + a.I, pol_w);
                    }
                    __syncwarp();
                    if (gather_lane)
                        tma_gather4(st + 2 * kTileBytesA + lane * 4 * kBK * 2, &tmX, &full_bar[stage], kb * kBK,
                                    tr[0], tr[1], tr[2], tr[3], pol_x);
                    if (++stage == kFStages) { stage = 0; phase ^= 1; }
                }
            } else {
                const int row = ft.e * a.H + ft.mb * 2 * kBM + ft.h0 * kBM;
                const uint32_t tx = (ft.two ? 2 : 1) * kTileBytesA + nbox * kBoxBytesB;
                // the weights of the first stages go out before the wait for act
                const int pre = KB_dn < kFStages ? KB_dn : kFStages;
                const int stage0 = stage;
                for (int kb = 0; kb < pre && ok; ++kb) {
                    if (lane == 0) {
                        ok = mbar_wait(&empty_bar[stage], phase ^ 1, abort_flag, a.err, 0);
                        if (ok) {
                            uint8_t *st = ring + stage * kFSlot;
                            mbar_arrive_expect_tx(&full_bar[stage], tx);
                            tma_load_2d(st, &tmWd, &full_bar[stage], kb * kBK, row, pol_w);
                            if (ft.two)
                                tma_load_2d(st + kTileBytesA, &tmWd, &full_bar[stage], kb * kBK, row + kBM, pol_w);
                        }
                    }
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (++stage == kFStages) { stage = 0; phase ^= 1; }
                }
                // act rows of expert e: every gate/up tile of e has finished (4 epilogue warps each)
                if (ok && lane == 0) ok = wait_count(a.gu_done + ft.e, 4u * MB_gu, abort_flag, a.err);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                if (lane == 0) {
                    fence_proxy_async_global();          // act was written by other threads' generic stores
                    for (int kb = 0; kb < pre; ++kb) {
                        const int s = (stage0 + kb) % kFStages;
                        uint8_t *sb = ring + s * kFSlot + 2 * kTileBytesA;
                        for (int b = 0; b < nbox; ++b)
                            tma_load_2d(sb + b * kBoxBytesB, &tmAct, &full_bar[s], kb * kBK, ft.row0 + b * kBoxN,
                                        pol_x);
                    }
                }
                for (int kb = pre; kb < KB_dn && ok; ++kb) {
                    if (lane == 0) {
                        ok = mbar_wait(&empty_bar[stage], phase ^ 1, abort_flag, a.err, 0);
                        if (ok) {
                            uint8_t *st = ring + stage * kFSlot;
                            mbar_arrive_expect_tx(&full_bar[stage], tx);
                            tma_load_2d(st, &tmWd, &full_bar[stage], kb * kBK, row, pol_w);
                            if (ft.two)
                                tma_load_2d(st + kTileBytesA, &tmWd, &full_bar[stage], kb * kBK, row + kBM, pol_w);
                            for (int b = 0; b < nbox; ++b)
                                tma_load_2d(st + 2 * kTileBytesA + b * kBoxBytesB, &tmAct, &full_bar[stage],
                                            kb * kBK, ft.row0 + b * kBoxN, pol_x);
                        }
                    }
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (++stage == kFStages) { stage = 0; phase ^= 1; }
                }
            }
            tile = static_cast<int>(__shfl_sync(0xffffffffu, next, 0));
        }
    } else if (warp == 1) {
        // ================================ MMA issuer ============================
        if (lane == 0) {
            int stage = 0, qs = 0, buf = 0;
            uint32_t phase = 0, qph = 0, bphase = 0;
            bool ok = true;
            while (ok) {
                int tile = -1;
                ok = pop_tile(fs, q_full, q_empty, qs, qph, abort_flag, a.err, tile);
                if (++qs == kFQueue) { qs = 0; qph ^= 1; }
                if (!ok || tile < 0) break;
                const FTile ft = fused_tile(tile, tc, fs, MB_gu, MB_dn, a.H);
                const uint32_t idesc = idesc_bf16_f32(kBM, ft.n_mma);
                ok = mbar_wait(&tempty_bar[buf], bphase ^ 1, abort_flag, a.err);
                if (!ok) break;
                tc_fence_after_sync();
                const uint32_t d0 = tmem_base + buf * kFAccCols;
                const int KB = ft.gu ? KB_gu : KB_dn;
                for (int kb = 0; kb < KB; ++kb) {
                    ok = mbar_wait(&full_bar[stage], phase, abort_flag, a.err, 0);
                    if (!ok) break;
                    tc_fence_after_sync();
                    const uint32_t st = smem_u32(ring + stage * kFSlot);
                    const uint64_t da0 = sw128_kmajor_desc(st), da1 = sw128_kmajor_desc(st + kTileBytesA);
                    const uint64_t db = sw128_kmajor_desc(st + 2 * kTileBytesA);
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k) {
                        const uint32_t acc = (kb | k) != 0;
                        umma_bf16_ss(d0, da0 + 2 * k, db + 2 * k, idesc, acc);
                        if (ft.two) umma_bf16_ss(d0 + kFBN, da1 + 2 * k, db + 2 * k, idesc, acc);
                    }
                    umma_commit(&empty_bar[stage]);
                    if (++stage == kFStages) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                umma_commit(&tfull_bar[buf]);
                if (++buf == 2) { buf = 0; bphase ^= 1; }
            }
            umma_commit(drain_bar);
            volatile int never = 0;
            mbar_wait(drain_bar, 0, &never, a.err);
        }
    } else if (warp < 6) {
        // ============================ warps 2-5: epilogue ========================
        const int q = warp & 3;
        int buf = 0, qs = 0;
        uint32_t bphase = 0, qph = 0;
        for (;;) {
            int tile = -1;
            bool ok = true;
            if (lane == 0) ok = pop_tile(fs, q_full, q_empty, qs, qph, abort_flag, a.err, tile);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            tile = __shfl_sync(0xffffffffu, tile, 0);
            if (++qs == kFQueue) { qs = 0; qph ^= 1; }
            if (!ok || tile < 0) break;
            const FTile ft = fused_tile(tile, tc, fs, MB_gu, MB_dn, a.H);
            if (!__shfl_sync(0xffffffffu, mbar_wait(&tfull_bar[buf], bphase, abort_flag, a.err, 128), 0)) break;
            tc_fence_after_sync();
            const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * kFAccCols;
            if (ft.gu) {
                const int f = ft.mb * kBM + q * 32 + lane;
                const bool f_ok = f < a.I;
                uint16_t *dst = a.act + static_cast<size_t>(ft.row0) * a.I + f;
                for (int c0 = 0; c0 < ft.n_mma; c0 += 16) {
                    uint32_t g[16], u[16];
                    tmem_ld_32x32b_x16(tb + c0, g);
                    tmem_ld_32x32b_x16(tb + kFBN + c0, u);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int n = c0 + j;
                        if (f_ok && n < ft.valid) {
                            float v = __uint_as_float(g[j]);
                            v = v / (1.0f + expf(-v)) * __uint_as_float(u[j]);
                            dst[static_cast<size_t>(n) * a.I] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
                        }
                    }
                }
            } else {
                for (int h = 0; h < (ft.two ? 2 : 1); ++h) {
                    const int f = ft.mb * 2 * kBM + (ft.h0 + h) * kBM + q * 32 + lane;
                    const bool f_ok = f < a.H;
                    uint16_t *dst = a.y + static_cast<size_t>(ft.row0) * a.H + f;
                    for (int c0 = 0; c0 < ft.n_mma; c0 += 16) {
                        uint32_t v[16];
                        tmem_ld_32x32b_x16(tb + h * kFBN + c0, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int n = c0 + j;
                            if (f_ok && n < ft.valid)
                                dst[static_cast<size_t>(n) * a.H] =
                                    __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[j])));
                        }
                    }
                }
            }
            tc_fence_before_sync();
            mbar_arrive(&tempty_bar[buf]);
            // the tile's rows are stored: count it (release), for the down tiles
            // of this expert (TMA reads of act) or for finalize
            if (ft.gu) fence_proxy_async_global();
            __syncwarp();
            if (lane == 0) red_release_add_u32(ft.gu ? a.gu_done + ft.e : a.dn_done, 1u);
            if (++buf == 2) { buf = 0; bphase ^= 1; }
        }
    }

    // ---- finalize: once every down tile has finished, on every CTA ---------------
    __syncthreads();
    griddep_launch_dependents();
    if (threadIdx.x == 0)
        wait_count(a.dn_done, 4u * static_cast<unsigned int>(tc.n_dn + tc.n_split), abort_flag, a.err);
    __syncthreads();
    if (!*abort_flag) {
        ld_acquire_u32(a.dn_done);
        const int vpr = a.H / 8;
        const long long total = static_cast<long long>(a.T) * vpr;
        const uint4 *y4 = reinterpret_cast<const uint4 *>(a.y);
        uint4 *out4 = reinterpret_cast<uint4 *>(a.out);
        for (long long i = blockIdx.x * static_cast<long long>(kFThreads) + threadIdx.x; i < total;
             i += static_cast<long long>(gridDim.x) * kFThreads) {
            const int t = static_cast<int>(i / vpr);
            const int v = static_cast<int>(i - static_cast<long long>(t) * vpr);
            // every slot's y row first (one L2 latency), then the sum in slot order
            uint4 yv[kFMaxSlots];
            float wv[kFMaxSlots];
#pragma unroll
            for (int j = 0; j < kFMaxSlots; ++j) {
                yv[j] = make_uint4(0u, 0u, 0u, 0u);
                wv[j] = 0.f;
                if (j < K) {
                    const int r = fs.inv[t * K + j];
                    wv[j] = fs.w[t * K + j];
                    if (r >= 0 && r < P) yv[j] = __ldcg(y4 + static_cast<size_t>(r) * vpr + v);
                    else if (v == 0) raise_error(a.err, kErrBadRow);
                }
            }
            float acc[8];
#pragma unroll
            for (int j = 0; j < kFMaxSlots; ++j) {
                if (j < K) {
                    const uint32_t qs[4] = {yv[j].x, yv[j].y, yv[j].z, yv[j].w};
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float x = bf16_bits_to_float((qs[e >> 1] >> ((e & 1) * 16)) & 0xFFFFu);
                        acc[e] = (j == 0) ? __fmul_rn(x, wv[j]) : __fmaf_rn(x, wv[j], acc[e]);
                    }
                }
            }
            uint4 o;
            uint32_t *op = &o.x;
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const __nv_bfloat16 lo = __float2bfloat16_rn(acc[2 * h]), hi = __float2bfloat16_rn(acc[2 * h + 1]);
                op[h] = static_cast<uint32_t>(__bfloat16_as_ushort(lo)) |
                        (static_cast<uint32_t>(__bfloat16_as_ushort(hi)) << 16);
            }
            out4[i] = o;
        }
    }
    __syncthreads();
    if (*abort_flag) {
        for (int i = 0; i < 1000; ++i) __nanosleep(1000);
    }
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, kFTmemCols);
    }
}

constexpr size_t kFBarBytes = 8 * (2 * kFStages + 4 + 2 * kFQueue + 1);
constexpr size_t kFSmemBytes = 1024 + static_cast<size_t>(kFStages) * kFSlot + kFBarBytes + 64 + sizeof(FusedSmem);
static_assert(kFSmemBytes + 64 <= kSmemLimit, "shared memory");
static_assert(kFMaxE <= kFThreads, "one scan thread per expert");
static_assert(kFMaxT <= 64, "token masks are 64 bits");
static_assert(kFTmemCols <= 512, "TMEM");

template <int PER_LANE>
cudaError_t launch_fused_t(const FusedArgs &a, const CUtensorMap (&m)[4], cudaStream_t s) {
    auto kern = fused_decode_kernel<PER_LANE>;
    cudaError_t st = ensure_dynamic_smem(kern, kFSmemBytes);
    if (st != cudaSuccess) return st;
    // one CTA per SM (the shared memory admits no second); tiles are handed
    // out dynamically, so no CTA needs another to be resident at the same time
    return launch_pdl(kern, dim3(num_sms()), dim3(kFThreads), kFSmemBytes, s, m[0], m[1], m[2], m[3], a);
}

}  // namespace

bool fused_decode_supported(int T, int H, int I, int E, int k, int S, int fmt) {
    return fmt == 0 && T >= 1 && T <= kFMaxT && k + S <= kFMaxSlots && E + S <= kFMaxE && E <= kFMaxE &&
           H % 8 == 0 && I % 8 == 0;
}

size_t fused_counter_words(int E, int S) { return static_cast<size_t>(E + S) + 3; }

cudaError_t launch_fused_decode(const float *logits, const uint16_t *hidden, const void *w_gu, const void *w_d,
                                int T, int H, int I, int E, int k, int S, int32_t *ids, float *w, int32_t *counts,
                                int32_t *offsets, int32_t *perm, int32_t *inv_perm, uint16_t *act, uint16_t *y,
                                uint16_t *out, unsigned int *done, int *err, cudaStream_t s) {
    if (!fused_decode_supported(T, H, I, E, k, S, 0)) return cudaErrorInvalidValue;
    const int Et = E + S, P = T * (k + S);
    CUtensorMap m[4];
    bool ok = make_map(&m[0], w_gu, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, static_cast<uint64_t>(Et) * 2 * I, kBK,
                       kBM, CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_map(&m[1], w_d, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, I, static_cast<uint64_t>(Et) * H, kBK, kBM,
                       CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_map(&m[2], hidden, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, T, kBK, 1, CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_map(&m[3], act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, I, P, kBK, kBoxN, CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok) return cudaErrorInvalidValue;
    // the counters start at zero on every call
    cudaError_t st = launch_pdl(fused_reset_kernel, dim3(1), dim3(32), 0, s, done,
                                static_cast<int>(fused_counter_words(E, S)));
    if (st != cudaSuccess) return st;
    FusedArgs a;
    a.logits = logits;
    a.T = T;
    a.E = E;
    a.k = k;
    a.S = S;
    a.H = H;
    a.I = I;
    a.ids = ids;
    a.counts = counts;
    a.offsets = offsets;
    a.perm = perm;
    a.inv_perm = inv_perm;
    a.w = w;
    a.act = act;
    a.y = y;
    a.out = out;
    a.gu_done = done;
    a.dn_done = done + Et;
    a.next_tile = done + Et + 1;
    a.routed = done + Et + 2;
    a.err = err;
    const int per_lane = (E + 31) / 32;
    if (per_lane <= 1) return launch_fused_t<1>(a, m, s);
    if (per_lane <= 2) return launch_fused_t<2>(a, m, s);
    if (per_lane <= 4) return launch_fused_t<4>(a, m, s);
    return launch_fused_t<8>(a, m, s);
}

}  // namespace moe
