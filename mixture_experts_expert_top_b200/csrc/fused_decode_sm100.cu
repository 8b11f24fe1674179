// fused_decode_sm100.cu -- the whole MoE layer for a decode batch (bf16
// weights) in one persistent kernel: routing, bucketing, the gate/up grouped
// GEMM with SwiGLU, the down grouped GEMM and the weighted finalize.
//
// The steps are the layer's (InfiniLM PR #500 Qwen3-MoE report §2.1-§2.2;
// FlashInfer PR #7196 analysis §1 for finalize, §2 for the runtime-N tiles;
// the GC-MoE abstract fuses the layer's steps into one graph). One launch, no
// host synchronisation and no kernel boundary between the steps:
//  - Every CTA routes and buckets the whole batch itself, in shared memory
//    (a decode batch is at most 64 tokens: the logits are 32 KB from L2), so
//    no CTA waits for another to learn the tile list. CTA 0 also writes the
//    routing and permutation to the workspace.
//  - Tiles: the gate/up tiles of every expert, then the down tiles, walked
//    blockIdx.x + i * gridDim.x by the same warp-specialised pipeline as the
//    weights-on-M kernel (warp 0 TMA, warp 1 MMA, warps 2-5 epilogue): gate/up
//    reads the token rows through perm (gather4), down reads act rows.
//  - A down tile of expert e reads act rows written by the gate/up tiles of
//    e, which may run on other CTAs: their epilogues count finished tiles per
//    expert in global memory (release), and the producer waits for the count
//    (acquire, bounded) before it loads act. Finalize waits likewise for the
//    count of finished down tiles, then every CTA combines a share of the
//    tokens in the finalize kernel's order of operations.
//  - The launch is cooperative, so every CTA is resident at once: a CTA
//    waits only for tiles that CTAs already running will finish, and every
//    CTA finishes its gate/up tiles before its down tiles. Every wait is
//    bounded (a timeout raises the device flag and the CTA unwinds).
#include "bucket_dev.cuh"
#include "gemm_common.cuh"
#include "launch_util.cuh"
#include "route_dev.cuh"

namespace moe {
namespace {

using namespace gemm;

constexpr int kFThreads = 256;          // 0 TMA, 1 MMA, 2-5 epilogue; all 8 warps route, bucket and finalize
constexpr int kFBN = 32;                // token rows per tile
constexpr int kFMaxT = 64;
constexpr int kFMaxSlots = 16;
constexpr int kFMaxP = kFMaxT * kFMaxSlots;
constexpr int kFMaxE = 256;
constexpr int kFStages = 5;
constexpr int kFGuStage = 2 * kTileBytesA + kFBN * kBK * 2;        // 36 KB: gate, up, token rows (K = 64)
constexpr int kFDnStage = 2 * (kTileBytesA + kFBN * kBK * 2);      // 40 KB: two K = 64 blocks of W_d and act
constexpr int kFSlot = kFDnStage;
constexpr int kFAccCols = 2 * kFBN;     // per buffer: g and u (down uses the first kFBN columns)
constexpr int kFTmemCols = 128;
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
    int *err;
};

struct FusedSmem {
    int32_t perm[kFMaxP];
    int32_t inv[kFMaxP];
    float w[kFMaxP];
    int off[kFMaxE + 1];
    int pre_gu[kFMaxE + 1];
    int pre_dn[kFMaxE + 1];
};

// Tile prefix over experts from offsets already in shared memory (every
// thread of the CTA calls it).
__device__ void tile_prefix_smem(const int *off, int E, int MB, int *pre) {
    if (threadIdx.x == 0) {
        int run = 0;
        pre[0] = 0;
        for (int e = 0; e < E; ++e) {
            run += ((off[e + 1] - off[e] + kFBN - 1) / kFBN) * MB;
            pre[e + 1] = run;
        }
    }
    __syncthreads();
}

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
        if (sleep_ns < 1024) sleep_ns <<= 1;
    }
    return true;
}

struct FTile {
    bool gu;        // gate/up tile (else down)
    TileInfo t;
};

__device__ __forceinline__ FTile fused_tile(int tile, int n_gu, const FusedSmem &fs, int E, int MB_gu, int MB_dn) {
    FTile f;
    f.gu = tile < n_gu;
    f.t = f.gu ? decode_tile(tile, fs.pre_gu, fs.off, E, MB_gu, kFBN)
               : decode_tile(tile - n_gu, fs.pre_dn, fs.off, E, MB_dn, kFBN);
    return f;
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
    uint64_t *drain_bar = tempty_bar + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain_bar + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
    FusedSmem &fs = *reinterpret_cast<FusedSmem *>(tmem_holder + 16);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int K = a.k + a.S, Et = a.E + a.S, P = a.T * K;
    const int MB_gu = (a.I + kBM - 1) / kBM, MB_dn = (a.H + kBM - 1) / kBM;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kFStages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull_bar[b], 1);
            mbar_init(&tempty_bar[b], kEpiThreads);
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
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, kFTmemCols);
        tmem_relinquish();
    }

    // ---- routing and bucketing of the whole batch, in shared memory ----------
    // (the ring is free until the tiles start: ids and the bucketing scratch live there)
    int32_t *ids_s = reinterpret_cast<int32_t *>(ring);                   // [P]
    int32_t *counts_s = ids_s + kFMaxP;                                   // [Et]
    int *bucket_scratch = counts_s + kFMaxE;                              // [(8 + 2) * Et]
    for (int t = warp; t < a.T; t += kFThreads / 32) {
        int id;
        float wt;
        route_token<PER_LANE>(a.logits + static_cast<size_t>(t) * a.E, a.E, a.k, id, wt);
        shared_slot(lane, a.k, a.E, id, wt);
        if (lane < K) {
            ids_s[t * K + lane] = id;
            fs.w[t * K + lane] = wt;
        }
    }
    __syncthreads();
    bucket_single_cta<kFThreads>(ids_s, P, Et, counts_s, fs.off, fs.perm, fs.inv, bucket_scratch, a.err);
    __syncthreads();
    if (blockIdx.x == 0) {
        for (int i = threadIdx.x; i < P; i += kFThreads) {
            a.ids[i] = ids_s[i];
            a.w[i] = fs.w[i];
            a.perm[i] = fs.perm[i];
            a.inv_perm[i] = fs.inv[i];
        }
        for (int e = threadIdx.x; e <= Et; e += kFThreads) {
            a.offsets[e] = fs.off[e];
            if (e < Et) a.counts[e] = counts_s[e];
        }
    }
    tile_prefix_smem(fs.off, Et, MB_gu, fs.pre_gu);
    tile_prefix_smem(fs.off, Et, MB_dn, fs.pre_dn);
    fence_proxy_async_smem();            // the ring's routing scratch is overwritten by TMA next
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_holder;
    const int n_gu = fs.pre_gu[Et], n_dn = fs.pre_dn[Et];
    const int total_tiles = n_gu + n_dn;
    // token row of permuted row r (rows past P read row 0; they are never stored)
    auto token_of = [&](int r) { return r < P ? fs.perm[r] / K : 0; };

    if (warp == 0) {
        // ================================ TMA producer ==========================
        const uint64_t pol_w = l2_policy_evict_first();
        const uint64_t pol_x = l2_policy_evict_last();
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
            const FTile ft = fused_tile(tile, n_gu, fs, Et, MB_gu, MB_dn);
            const TileInfo &ti = ft.t;
            const int nbox = ti.n_mma / kBoxN;
            if (ft.gu) {
                const int a_row = ti.e * 2 * a.I + ti.mb * kBM;
                const uint32_t tx = 2 * kTileBytesA + nbox * kBoxBytesB;
                const bool gather_lane = 4 * lane < ti.n_mma;
                int tr[4] = {0, 0, 0, 0};
                if (gather_lane) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) tr[j] = token_of(ti.row0 + 4 * lane + j);
                }
                const int KB = (a.H + kBK - 1) / kBK;
                for (int kb = 0; kb < KB; ++kb) {
                    if (lane == 0) ok = mbar_wait(&empty_bar[stage], phase ^ 1, abort_flag, a.err, 0);
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    uint8_t *st = ring + stage * kFSlot;
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&full_bar[stage], tx);
                        tma_load_2d(st, &tmWgu, &full_bar[stage], kb * kBK, a_row, pol_w);
                        tma_load_2d(st + kTileBytesA, &tmWgu, &full_bar[stage], kb * kBK, a_row + a.I, pol_w);
                    }
                    __syncwarp();
                    if (gather_lane)
                        tma_gather4(st + 2 * kTileBytesA + lane * 4 * kBK * 2, &tmX, &full_bar[stage], kb * kBK, tr[0],
                                    tr[1], tr[2], tr[3], pol_x);
                    if (++stage == kFStages) { stage = 0; phase ^= 1; }
                }
            } else {
                // act rows of expert e: every gate/up tile of e has finished (4 epilogue warps each)
                const int cnt = fs.off[ti.e + 1] - fs.off[ti.e];
                const unsigned int need = 4u * MB_gu * ((cnt + kFBN - 1) / kFBN);
                if (lane == 0) ok = wait_count(a.gu_done + ti.e, need, abort_flag, a.err);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                fence_proxy_async_global();              // act was written by other threads' generic stores
                const int a_row = ti.e * a.H + ti.mb * kBM;
                const uint32_t tx = 2 * (kTileBytesA + nbox * kBoxBytesB);
                const int KB = (a.I + 2 * kBK - 1) / (2 * kBK);
                for (int kb = 0; kb < KB; ++kb) {
                    if (lane == 0) ok = mbar_wait(&empty_bar[stage], phase ^ 1, abort_flag, a.err, 0);
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    uint8_t *st = ring + stage * kFSlot;
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&full_bar[stage], tx);
                        for (int u = 0; u < 2; ++u) {
                            uint8_t *su = st + u * (kTileBytesA + kFBN * kBK * 2);
                            const int x = (2 * kb + u) * kBK;
                            tma_load_2d(su, &tmWd, &full_bar[stage], x, a_row, pol_w);
                            for (int b = 0; b < nbox; ++b)
                                tma_load_2d(su + kTileBytesA + b * kBoxBytesB, &tmAct, &full_bar[stage], x,
                                            ti.row0 + b * kBoxN, pol_x);
                        }
                    }
                    __syncwarp();
                    if (++stage == kFStages) { stage = 0; phase ^= 1; }
                }
            }
        }
    } else if (warp == 1) {
        // ================================ MMA issuer ============================
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int buf = 0;
            uint32_t bphase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
                const FTile ft = fused_tile(tile, n_gu, fs, Et, MB_gu, MB_dn);
                const uint32_t idesc = idesc_bf16_f32(kBM, ft.t.n_mma);
                ok = mbar_wait(&tempty_bar[buf], bphase ^ 1, abort_flag, a.err);
                if (!ok) break;
                tc_fence_after_sync();
                const uint32_t d0 = tmem_base + buf * kFAccCols;
                const int KB = ft.gu ? (a.H + kBK - 1) / kBK : (a.I + 2 * kBK - 1) / (2 * kBK);
                for (int kb = 0; kb < KB; ++kb) {
                    ok = mbar_wait(&full_bar[stage], phase, abort_flag, a.err, 0);
                    if (!ok) break;
                    tc_fence_after_sync();
                    const uint32_t st = smem_u32(ring + stage * kFSlot);
                    if (ft.gu) {
                        const uint64_t dg = sw128_kmajor_desc(st), du = sw128_kmajor_desc(st + kTileBytesA);
                        const uint64_t db = sw128_kmajor_desc(st + 2 * kTileBytesA);
#pragma unroll
                        for (int k = 0; k < kBK / 16; ++k) {
                            const uint32_t acc = (kb | k) != 0;
                            umma_bf16_ss(d0, dg + 2 * k, db + 2 * k, idesc, acc);
                            umma_bf16_ss(d0 + kFBN, du + 2 * k, db + 2 * k, idesc, acc);
                        }
                    } else {
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const uint32_t su = st + u * (kTileBytesA + kFBN * kBK * 2);
                            const uint64_t da = sw128_kmajor_desc(su), db = sw128_kmajor_desc(su + kTileBytesA);
#pragma unroll
                            for (int k = 0; k < kBK / 16; ++k)
                                umma_bf16_ss(d0, da + 2 * k, db + 2 * k, idesc, (kb | u | k) != 0);
                        }
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
        int buf = 0;
        uint32_t bphase = 0;
        for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
            const FTile ft = fused_tile(tile, n_gu, fs, Et, MB_gu, MB_dn);
            const TileInfo &ti = ft.t;
            if (!__shfl_sync(0xffffffffu, mbar_wait(&tfull_bar[buf], bphase, abort_flag, a.err, 128), 0)) break;
            tc_fence_after_sync();
            const int m_out = ft.gu ? a.I : a.H;
            const int f = ti.mb * kBM + q * 32 + lane;
            const bool f_ok = f < m_out;
            uint16_t *dst = (ft.gu ? a.act : a.y) + static_cast<size_t>(ti.row0) * m_out + f;
            const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * kFAccCols;
            for (int c0 = 0; c0 < ti.n_mma; c0 += 16) {
                uint32_t g[16], u[16];
                tmem_ld_32x32b_x16(tb + c0, g);
                if (ft.gu) tmem_ld_32x32b_x16(tb + kFBN + c0, u);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int n = c0 + j;
                    if (f_ok && n < ti.valid) {
                        float v = __uint_as_float(g[j]);
                        if (ft.gu) v = v / (1.0f + expf(-v)) * __uint_as_float(u[j]);
                        dst[static_cast<size_t>(n) * m_out] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
                    }
                }
            }
            tc_fence_before_sync();
            mbar_arrive(&tempty_bar[buf]);
            // the tile's rows are stored: count it (release), for the down tiles
            // of this expert (TMA reads of act) or for finalize
            if (ft.gu) fence_proxy_async_global();
            __syncwarp();
            if (lane == 0) red_release_add_u32(ft.gu ? a.gu_done + ti.e : a.dn_done, 1u);
            if (++buf == 2) { buf = 0; bphase ^= 1; }
        }
    }

    // ---- finalize: once every down tile has finished, on every CTA ---------------
    __syncthreads();
    if (threadIdx.x == 0) wait_count(a.dn_done, 4u * static_cast<unsigned int>(n_dn), abort_flag, a.err);
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
            float acc[8];
            for (int j = 0; j < K; ++j) {
                const int r = fs.inv[t * K + j];
                const float wj = fs.w[t * K + j];
                uint4 qv = make_uint4(0u, 0u, 0u, 0u);
                if (r >= 0 && r < P) qv = __ldcg(y4 + static_cast<size_t>(r) * vpr + v);
                else if (v == 0) raise_error(a.err, kErrBadRow);
                const uint32_t qs[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float x = bf16_bits_to_float((qs[e >> 1] >> ((e & 1) * 16)) & 0xFFFFu);
                    acc[e] = (j == 0) ? __fmul_rn(x, wj) : __fmaf_rn(x, wj, acc[e]);
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

constexpr size_t kFSmemBytes = 1024 + static_cast<size_t>(kFStages) * kFSlot + 8 * (2 * kFStages + 5) + 64 +
                               sizeof(FusedSmem);
static_assert(kFSmemBytes + 64 <= kSmemLimit, "shared memory");
static_assert(kFGuStage <= kFSlot, "a gate/up stage fits a ring slot");
// routing scratch in the ring: ids, counts, and the bucketing's (8 + 2) x E histograms
static_assert((kFMaxP + kFMaxE + 10 * kFMaxE) * 4 <= kFStages * kFSlot, "routing scratch fits the ring");

template <int PER_LANE>
cudaError_t launch_fused_t(const FusedArgs &a, const CUtensorMap (&m)[4], cudaStream_t s) {
    auto kern = fused_decode_kernel<PER_LANE>;
    cudaError_t st = ensure_dynamic_smem(kern, kFSmemBytes);
    if (st != cudaSuccess) return st;
    int dev = 0, blocks_per_sm = 0;
    if ((st = cudaGetDevice(&dev)) != cudaSuccess) return st;
    if ((st = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks_per_sm, kern, kFThreads, kFSmemBytes)) !=
        cudaSuccess)
        return st;
    if (blocks_per_sm < 1) return cudaErrorInvalidConfiguration;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(num_sms());           // one CTA per SM, all resident (cooperative launch)
    cfg.blockDim = dim3(kFThreads);
    cfg.dynamicSmemBytes = kFSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, m[0], m[1], m[2], m[3], a);
}

}  // namespace

bool fused_decode_supported(int T, int H, int I, int E, int k, int S, int fmt) {
    return fmt == 0 && T >= 1 && T <= kFMaxT && k + S <= kFMaxSlots && E + S <= kFMaxE && E <= kFMaxE &&
           H % 8 == 0 && I % 8 == 0;
}

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
    // the completion counters start at zero on every call
    cudaError_t st = cudaMemsetAsync(done, 0, sizeof(unsigned int) * (Et + 1), s);
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
    a.err = err;
    const int per_lane = (E + 31) / 32;
    if (per_lane <= 1) return launch_fused_t<1>(a, m, s);
    if (per_lane <= 2) return launch_fused_t<2>(a, m, s);
    if (per_lane <= 4) return launch_fused_t<4>(a, m, s);
    return launch_fused_t<8>(a, m, s);
}

}  // namespace moe
