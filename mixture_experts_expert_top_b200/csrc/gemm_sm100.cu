// gemm_sm100.cu -- grouped GEMMs of the MoE layer on sm_100a tensor cores.
//
// What they compute (InfiniLM PR #500 Qwen3-MoE report, §2.2 step 2: one
// grouped GEMM call covers every expert's slab of permuted rows):
//   gate/up:  act[r, i] = bf16( silu(g) * u ),  g = a[r] . W_gu[e, i],
//             u = a[r] . W_gu[e, I + i]   (fp32 accumulation, SwiGLU fused)
//   down:     y[r, h]  = bf16( act[r] . W_d[e, h] )
// for every permuted row r of expert e (offsets[e] <= r < offsets[e+1]).
//
// Design (sm_100a; the FlashInfer PR #7196 analysis §2 and the GC-MoE
// abstract describe the same operand roles):
//  - Weights are the MMA's A operand (M = 128 weight rows per tile), tokens
//    are the B operand (N = tokens). The MMA's N is chosen per tile at run
//    time as the routed-token count rounded up to 16, so a decode tile with 5
//    tokens issues N = 16 instructions and loads only 16 token rows.
//  - gate/up tiles hold 128 gate rows and the matching 128 up rows: two MMAs
//    per K step into two TMEM accumulators, so each epilogue thread finds g
//    and u of the same (feature, token) in the same TMEM lane.
//  - Persistent CTAs (one per SM) walk a static list of (expert, feature
//    block, token block) tiles; experts with no tokens have no tiles.
//  - Warp roles: warp 0 issues TMA loads into a STAGES-deep shared-memory
//    ring, warp 1 issues tcgen05.mma (one thread) and owns the TMEM
//    allocation, warps 2-5 drain the double-buffered TMEM accumulators
//    (tcgen05.ld), apply SwiGLU and store bf16 rows.
//  - W4A16 has a kernel of its own (grouped_gemm_int4_kernel): one ring stage
//    covers K = 256, so each packed weight row arrives as one 128-byte TMA
//    row; four groups of decode warps each turn one 64-K quarter of the stage
//    into bf16 (w = bf16(q * scale)) and store it straight into a TMEM ring,
//    from which the MMA reads its A operand. Shared memory carries 0.5 byte
//    per weight instead of the 4.5 bytes a decode through shared memory would
//    move (packed in, bf16 out, bf16 read again by the MMA).
//  - Every wait is bounded (see mbar_wait); a timeout raises the device flag
//    and unwinds the CTA.
#include "gemm_common.cuh"
#include "launch_util.cuh"

namespace moe {
namespace {

using namespace gemm;

// =============================================================================
// bf16 weights
// =============================================================================

// KSUB 64-K sub-blocks per ring stage: fewer, larger hand-offs between the
// producer and the MMA issuer. A stage holds, per sub-block u, the weight
// tile (gate/up: the gate tile then the up tile) and then all token tiles.
template <int BN, int STAGES, bool SWIGLU, int KSUB = 1>
struct Bf16Cfg {
    static constexpr int kNumA = (SWIGLU ? 2 : 1) * KSUB;
    static constexpr int kThreads = 192;
    static constexpr int kABytes = kNumA * kTileBytesA;
    static constexpr int kBSub = BN * kBK * 2;                 // token rows of one 64-K sub-block
    static constexpr int kStageBytes = kABytes + KSUB * kBSub;
    static constexpr int kAccCols = SWIGLU ? 2 * BN : BN;
    static constexpr int kTmemUsed = 2 * kAccCols;
    static constexpr int kTmemCols = kTmemUsed <= 32 ? 32 : kTmemUsed <= 64 ? 64 : kTmemUsed <= 128 ? 128
                                   : kTmemUsed <= 256 ? 256 : 512;
    static constexpr int kRingBytes = STAGES * kStageBytes;
    static constexpr int kNumBars = 2 * STAGES + 2 + 2 + 1;
    static constexpr int kSmemBytes = 1024 + kRingBytes + 8 * kNumBars + 64 + 2 * (kMaxExperts + 1) * 4;
    static_assert(kStageBytes % 1024 == 0, "tiles must keep 1024-byte alignment");
    static_assert(kTmemUsed <= 512, "TMEM holds 512 32-bit columns");
    static_assert(BN % kBoxN == 0 && BN <= 256, "BN");
    static_assert(kSmemBytes + 64 <= kSmemLimit, "shared memory");
};

template <int BN, int STAGES, bool SWIGLU, int KSUB>
__global__ void __launch_bounds__(192, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const Params p) {
    using C = Bf16Cfg<BN, STAGES, SWIGLU, KSUB>;
    extern __shared__ uint8_t smem_raw[];
    // operand tiles need 1024-byte alignment in the shared window (swizzle atoms)
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *ring = smem;                                    // STAGES x [A0 | A1 | B]
    uint64_t *bars = reinterpret_cast<uint64_t *>(ring + C::kRingBytes);
    uint64_t *full_bar = bars;                               // TMA -> MMA
    uint64_t *empty_bar = full_bar + STAGES;                 // MMA -> TMA
    uint64_t *tfull_bar = empty_bar + STAGES;                // MMA -> epilogue, 2 buffers
    uint64_t *tempty_bar = tfull_bar + 2;                    // epilogue -> MMA, 2 buffers
    uint64_t *drain_bar = tempty_bar + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain_bar + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
    int *off_s = reinterpret_cast<int *>(tmem_holder + 16);  // [E+1]
    int *pre_s = off_s + (kMaxExperts + 1);                  // [E+1] tile prefix

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int E = p.E;
    const int MB = (p.m_out + kBM - 1) / kBM;
    const int KB = (p.K + KSUB * kBK - 1) / (KSUB * kBK);   // ring stages per tile

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
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
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, C::kTmemCols);
        tmem_relinquish();
    }
    // barriers, tensor maps and TMEM are set up while the previous kernel drains
    const bool early = (p.hints & kGemmHintOffsetsReady) && !p.perm;
    if (!early) {
        if (warp == 0 && lane == 0 && (p.hints & kGemmHintPrefetchGuess)) {
            // the tile this CTA gets if every expert has rows and one token block
            const int e = blockIdx.x / MB, mb = blockIdx.x % MB;
            if (e < E) {
                const int a_row = e * p.w_rows + mb * kBM;
                for (int kb = 0; kb < KB && kb < kGuessKBlocks; ++kb) {
                    tma_prefetch_l2_2d(&tmA, kb * kBK, a_row);
                    if (SWIGLU) tma_prefetch_l2_2d(&tmA, kb * kBK, a_row + p.m_out);
                }
            }
        }
        griddep_wait();
    }
    build_tile_prefix<C::kThreads>(p.offsets, E, MB, BN, off_s, pre_s, p.P, p.err);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_holder;
    const int total_tiles = pre_s[E];

    if (warp == 0) {
        // ================================ TMA producer ==========================
        // Lane 0 runs the ring; with perm, lanes i < n_mma/4 issue the token
        // rows as gather4 loads (tile rows 4i .. 4i+3) straight from hidden.
        const uint64_t pol_w = p.evict_first_weights ? l2_policy_evict_first() : l2_policy_evict_last();
        const uint64_t pol_x = l2_policy_evict_last();
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        // early: the weight tiles of the first STAGES ring slots go out before
        // the previous kernel has finished; their token tiles follow the wait
        int preloaded = 0;
        if (early) {
            for (int tile = blockIdx.x; tile < total_tiles && preloaded < STAGES; tile += gridDim.x) {
                const TileInfo ti = decode_tile(tile, pre_s, off_s, E, MB, BN);
                const int a_row = ti.e * p.w_rows + ti.mb * kBM;
                const uint32_t tx = C::kABytes + KSUB * (ti.n_mma / kBoxN) * kBoxBytesB;
                for (int kb = 0; kb < KB && preloaded < STAGES; ++kb, ++preloaded) {
                    if (lane == 0) {
                        uint8_t *st = ring + preloaded * C::kStageBytes;
                        mbar_arrive_expect_tx(&full_bar[preloaded], tx);
                        for (int u = 0; u < KSUB; ++u) {
                            uint8_t *sa = st + (SWIGLU ? 2 * u : u) * kTileBytesA;
                            const int x = (kb * KSUB + u) * kBK;
                            tma_load_2d(sa, &tmA, &full_bar[preloaded], x, a_row, pol_w);
                            if (SWIGLU) tma_load_2d(sa + kTileBytesA, &tmA, &full_bar[preloaded], x, a_row + p.m_out, pol_w);
                        }
                    }
                }
            }
            griddep_wait();
        }
        int it = 0;
        for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
            const TileInfo ti = decode_tile(tile, pre_s, off_s, E, MB, BN);
            const int nbox = ti.n_mma / kBoxN;
            const int a_row = ti.e * p.w_rows + ti.mb * kBM;
            const uint32_t tx = C::kABytes + KSUB * nbox * kBoxBytesB;
            const bool gather_lane = p.perm && 4 * lane < ti.n_mma;
            int tr[4] = {0, 0, 0, 0};
            if (gather_lane) {
#pragma unroll
                for (int j = 0; j < 4; ++j) tr[j] = token_row(p, ti.row0 + 4 * lane + j);
            }
            for (int kb = 0; kb < KB; ++kb, ++it) {
                if (lane == 0) ok = mbar_wait(&empty_bar[stage], phase ^ 1, abort_flag, p.err, 0);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                uint8_t *st = ring + stage * C::kStageBytes;
                uint8_t *sb = st + C::kABytes;
                if (lane == 0) {
                    if (it >= preloaded) {
                        mbar_arrive_expect_tx(&full_bar[stage], tx);
                        for (int u = 0; u < KSUB; ++u) {
                            uint8_t *sa = st + (SWIGLU ? 2 * u : u) * kTileBytesA;
                            const int x = (kb * KSUB + u) * kBK;
                            tma_load_2d(sa, &tmA, &full_bar[stage], x, a_row, pol_w);
                            if (SWIGLU) tma_load_2d(sa + kTileBytesA, &tmA, &full_bar[stage], x, a_row + p.m_out, pol_w);
                        }
                    }
                    if (!p.perm)
                        for (int u = 0; u < KSUB; ++u)
                            for (int b = 0; b < nbox; ++b)
                                tma_load_2d(sb + u * C::kBSub + b * kBoxBytesB, &tmB, &full_bar[stage],
                                            (kb * KSUB + u) * kBK, ti.row0 + b * kBoxN, pol_x);
                }
                __syncwarp();
                if (gather_lane)
                    for (int u = 0; u < KSUB; ++u)
                        tma_gather4(sb + u * C::kBSub + lane * 4 * kBK * 2, &tmB, &full_bar[stage],
                                    (kb * KSUB + u) * kBK, tr[0], tr[1], tr[2], tr[3], pol_x);
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
        }
    } else if (warp == 1) {
        // ================================ MMA issuer ============================
        if (early) griddep_wait();
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int buf = 0;
            uint32_t bphase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
                const TileInfo ti = decode_tile(tile, pre_s, off_s, E, MB, BN);
                const uint32_t idesc = idesc_bf16_f32(kBM, ti.n_mma);
                ok = mbar_wait(&tempty_bar[buf], bphase ^ 1, abort_flag, p.err);
                if (!ok) break;
                tc_fence_after_sync();
                const uint32_t d0 = tmem_base + buf * C::kAccCols;
                for (int kb = 0; kb < KB; ++kb) {
                    ok = mbar_wait(&full_bar[stage], phase, abort_flag, p.err, 0);
                    if (!ok) break;
                    tc_fence_after_sync();
                    const uint32_t st = smem_u32(ring + stage * C::kStageBytes);
#pragma unroll
                    for (int u = 0; u < KSUB; ++u) {
                        const uint32_t sa = st + (SWIGLU ? 2 * u : u) * kTileBytesA;
                        const uint64_t da0 = sw128_kmajor_desc(sa);
                        const uint64_t db = sw128_kmajor_desc(st + C::kABytes + u * C::kBSub);
#pragma unroll
                        for (int k = 0; k < kBK / 16; ++k) {
                            const uint32_t acc = (kb | u | k) != 0;
                            // +32 bytes per K step inside the swizzled row: +2 in the >>4 address field
                            umma_bf16_ss(d0, da0 + 2 * k, db + 2 * k, idesc, acc);
                            if (SWIGLU) umma_bf16_ss(d0 + BN, sw128_kmajor_desc(sa + kTileBytesA) + 2 * k, db + 2 * k, idesc, acc);
                        }
                    }
                    umma_commit(&empty_bar[stage]);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                umma_commit(&tfull_bar[buf]);
                if (++buf == 2) { buf = 0; bphase ^= 1; }
            }
            // all issued MMAs complete before TMEM is released
            umma_commit(drain_bar);
            volatile int never = 0;
            mbar_wait(drain_bar, 0, &never, p.err);
        }
    } else {
        if (early) griddep_wait();
        run_epilogue<BN, SWIGLU, C::kAccCols>(p, pre_s, off_s, total_tiles, MB, tmem_base, tfull_bar, tempty_bar,
                                              abort_flag, 128);
    }

    // every role is done: the next kernel may start its set-up now
    griddep_launch_dependents();
    __syncthreads();
    if (*abort_flag) {
        // let copies already in flight land before the CTA's memory is reused
        for (int i = 0; i < 1000; ++i) __nanosleep(1000);
    }
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

// =============================================================================
// W4A16: int4 weights (one bf16 scale per 128 K), bf16 tokens
// =============================================================================

// GROUPS hand-off groups of decode warps: the 16 decode warps convert the
// four 64-K quarters of a stage (one quarter per 4 warps, one warp per TMEM
// lane quarter), and the quarters of one group share one TMEM ring slot, so
// the MMA issuer is signalled GROUPS times per stage, not four.
template <int BN, int STAGES, bool SWIGLU, int GROUPS = kConvGroups>
struct Int4Cfg {
    static_assert(kQuarters % GROUPS == 0, "groups split the four quarters evenly");
    static constexpr int kQPG = kQuarters / GROUPS;                     // quarters per group (slot)
    static constexpr int kNumA = SWIGLU ? 2 : 1;
    static constexpr int kThreads = 192 + 128 * kConvGroups;
    static constexpr int kABytes = kNumA * kPackedTile;                 // packed A per stage (K = 256)
    static constexpr int kBQuarter = BN * kBK * 2;                      // token rows for one 64-K quarter
    static constexpr int kStageBytes = kABytes + kQuarters * kBQuarter;
    static constexpr int kAccCols = SWIGLU ? 2 * BN : BN;
    static constexpr int kACols = kNumA * (kBK / 2);                    // TMEM columns per decoded quarter
    static constexpr int kSlotCols = kQPG * kACols;                     // TMEM columns per ring slot
    static constexpr int kTmemAStages = (512 - 2 * kAccCols) / kSlotCols < kMaxTmemA
                                            ? (512 - 2 * kAccCols) / kSlotCols
                                            : kMaxTmemA;
    static constexpr int kTmemUsed = 2 * kAccCols + kTmemAStages * kSlotCols;
    static constexpr int kTmemCols = kTmemUsed <= 32 ? 32 : kTmemUsed <= 64 ? 64 : kTmemUsed <= 128 ? 128
                                   : kTmemUsed <= 256 ? 256 : 512;
    static constexpr int kRingBytes = STAGES * kStageBytes;
    static constexpr int kNumBars = 2 * STAGES + 2 * kMaxTmemA + 2 + 2 + 1;
    static constexpr int kSmemBytes = 1024 + kRingBytes + 8 * kNumBars + 64 + 2 * (kMaxExperts + 1) * 4;
    static_assert(kStageBytes % 1024 == 0 && kBQuarter % 1024 == 0, "tiles must keep 1024-byte alignment");
    static_assert(kTmemUsed <= 512, "TMEM holds 512 32-bit columns");
    static_assert(kTmemAStages >= GROUPS, "every decode group needs a TMEM slot in flight");
    static_assert(BN % kBoxN == 0 && BN <= 256, "BN");
    static_assert(kSmemBytes + 64 <= kSmemLimit, "shared memory");
};

template <int BN, int STAGES, bool SWIGLU, int GROUPS>
__global__ void __launch_bounds__(Int4Cfg<BN, STAGES, SWIGLU, GROUPS>::kThreads, 1)
grouped_gemm_int4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                         const Params p) {
    using C = Int4Cfg<BN, STAGES, SWIGLU, GROUPS>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *ring = smem;                                    // STAGES x [Aq0 | Aq1 | B quarter 0..3]
    uint64_t *bars = reinterpret_cast<uint64_t *>(ring + C::kRingBytes);
    uint64_t *full_bar = bars;                               // TMA -> decode groups
    uint64_t *empty_bar = full_bar + STAGES;                 // MMA -> TMA
    uint64_t *tready_bar = empty_bar + STAGES;               // decode group -> MMA (TMEM ring slot)
    uint64_t *tfree_bar = tready_bar + kMaxTmemA;            // MMA -> decode groups
    uint64_t *tfull_bar = tfree_bar + kMaxTmemA;             // MMA -> epilogue, 2 buffers
    uint64_t *tempty_bar = tfull_bar + 2;                    // epilogue -> MMA, 2 buffers
    uint64_t *drain_bar = tempty_bar + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain_bar + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
    int *off_s = reinterpret_cast<int *>(tmem_holder + 16);  // [E+1]
    int *pre_s = off_s + (kMaxExperts + 1);                  // [E+1] tile prefix

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int E = p.E;
    const int MB = (p.m_out + kBM - 1) / kBM;
    const int KS = (p.K + 4 * kBK - 1) / (4 * kBK);          // stages of K = 256 per tile

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int t = 0; t < C::kTmemAStages; ++t) {
            mbar_init(&tready_bar[t], 128 * C::kQPG);   // every warp of one decode group
            mbar_init(&tfree_bar[t], 1);
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
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, C::kTmemCols);
        tmem_relinquish();
    }
    // barriers, tensor maps and TMEM are set up while the previous kernel drains
    griddep_wait();
    build_tile_prefix<C::kThreads>(p.offsets, E, MB, BN, off_s, pre_s, p.P, p.err);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_holder;
    const uint32_t tmem_a0 = tmem_base + 2 * C::kAccCols;   // first decoded-A column
    const int total_tiles = pre_s[E];

    if (warp == 0) {
        // ================================ TMA producer ==========================
        const uint64_t pol_w = p.evict_first_weights ? l2_policy_evict_first() : l2_policy_evict_last();
        const uint64_t pol_x = l2_policy_evict_last();
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
            const TileInfo ti = decode_tile(tile, pre_s, off_s, E, MB, BN);
            const int nbox = ti.n_mma / kBoxN;
            const int a_row = ti.e * p.w_rows + ti.mb * kBM;
            const uint32_t tx = C::kABytes + kQuarters * nbox * kBoxBytesB;
            const bool gather_lane = p.perm && 4 * lane < ti.n_mma;
            int tr[4] = {0, 0, 0, 0};
            if (gather_lane) {
#pragma unroll
                for (int j = 0; j < 4; ++j) tr[j] = token_row(p, ti.row0 + 4 * lane + j);
            }
            for (int ks = 0; ks < KS; ++ks) {
                if (lane == 0) ok = mbar_wait(&empty_bar[stage], phase ^ 1, abort_flag, p.err, 256);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                uint8_t *st = ring + stage * C::kStageBytes;
                uint8_t *sb = st + C::kABytes;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&full_bar[stage], tx);
                    tma_load_2d(st, &tmA, &full_bar[stage], ks * 128, a_row, pol_w);
                    if (SWIGLU) tma_load_2d(st + kPackedTile, &tmA, &full_bar[stage], ks * 128, a_row + p.m_out, pol_w);
                    if (!p.perm)
                        for (int j = 0; j < kQuarters; ++j)
                            for (int b = 0; b < nbox; ++b)
                                tma_load_2d(sb + j * C::kBQuarter + b * kBoxBytesB, &tmB, &full_bar[stage],
                                            (ks * kQuarters + j) * kBK, ti.row0 + b * kBoxN, pol_x);
                }
                __syncwarp();
                if (gather_lane)
                    for (int j = 0; j < kQuarters; ++j)
                        tma_gather4(sb + j * C::kBQuarter + lane * 4 * kBK * 2, &tmB, &full_bar[stage],
                                    (ks * kQuarters + j) * kBK, tr[0], tr[1], tr[2], tr[3], pol_x);
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
        }
    } else if (warp == 1) {
        // ================================ MMA issuer ============================
        if (lane == 0) {
            int stage = 0;
            uint32_t phase_unused = 0;
            (void)phase_unused;
            int t = 0;                  // TMEM ring slot of the next quarter
            uint32_t tphase = 0;
            int buf = 0;
            uint32_t bphase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
                const TileInfo ti = decode_tile(tile, pre_s, off_s, E, MB, BN);
                const uint32_t idesc = idesc_bf16_f32(kBM, ti.n_mma);
                ok = mbar_wait(&tempty_bar[buf], bphase ^ 1, abort_flag, p.err);
                if (!ok) break;
                tc_fence_after_sync();
                const uint32_t d0 = tmem_base + buf * C::kAccCols;
                for (int ks = 0; ks < KS && ok; ++ks) {
                    const uint32_t sb = smem_u32(ring + stage * C::kStageBytes + C::kABytes);
                    for (int g = 0; g < GROUPS; ++g) {
                        // tready implies the stage's TMA data landed (the decode group waited for it)
                        ok = mbar_wait(&tready_bar[t], tphase, abort_flag, p.err, 0);
                        if (!ok) break;
                        tc_fence_after_sync();
#pragma unroll
                        for (int qq = 0; qq < C::kQPG; ++qq) {
                            const int j = g * C::kQPG + qq;                     // quarter of the stage
                            const uint32_t a0 = tmem_a0 + t * C::kSlotCols + qq * C::kACols;
                            const uint64_t db = sw128_kmajor_desc(sb + j * C::kBQuarter);
#pragma unroll
                            for (int k = 0; k < kBK / 16; ++k) {
                                const uint32_t acc = (ks | j | k) != 0;
                                // 16 K elements = 8 TMEM columns of A; +32 bytes of B per K step
                                umma_bf16_ts(d0, a0 + 8 * k, db + 2 * k, idesc, acc);
                                if (SWIGLU) umma_bf16_ts(d0 + BN, a0 + 32 + 8 * k, db + 2 * k, idesc, acc);
                            }
                        }
                        umma_commit(&tfree_bar[t]);
                        if (++t == C::kTmemAStages) { t = 0; tphase ^= 1; }
                    }
                    if (!ok) break;
                    umma_commit(&empty_bar[stage]);
                    if (++stage == STAGES) stage = 0;
                }
                if (!ok) break;
                umma_commit(&tfull_bar[buf]);
                if (++buf == 2) { buf = 0; bphase ^= 1; }
            }
            umma_commit(drain_bar);
            volatile int never = 0;
            mbar_wait(drain_bar, 0, &never, p.err);
        }
    } else if (warp < 6) {
        run_epilogue<BN, SWIGLU, C::kAccCols>(p, pre_s, off_s, total_tiles, MB, tmem_base, tfull_bar, tempty_bar,
                                              abort_flag);
    } else {
        // ====== warps 6-21: quarter g of every ring stage =======================
        // Row r of the tile, packed bytes [32g, 32g+32) of the stage's 128-byte
        // row (stored with the 128-byte swizzle: 16-byte chunk c of row r sits
        // at chunk c ^ (r % 8)), K elements 64g .. 64g+63 of the stage. The
        // quarter belongs to hand-off group g / kQPG, column block g % kQPG of
        // that group's TMEM slot.
        const int g = (warp - 6) >> 2;
        const int grp_id = g / C::kQPG;
        const uint32_t qcol = static_cast<uint32_t>((g % C::kQPG) * C::kACols);
        const int q = warp & 3;                 // TMEM lane quarter = rows q*32 .. q*32+31
        const int r = q * 32 + lane;
        const int kgroups = p.K / 128;
        const size_t srows = static_cast<size_t>(p.E) * p.w_rows;
        // position of the next stage to decode: tile n_tile, stage ks n_ks
        int n_tile = blockIdx.x, n_ks = 0;
        const uint16_t *n_srow[2] = {nullptr, nullptr};   // scale rows of n_tile
        auto set_rows = [&]() {
            n_srow[0] = n_srow[1] = nullptr;
            if (n_tile >= total_tiles) return;
            const TileInfo ti = decode_tile(n_tile, pre_s, off_s, E, MB, BN);
            const size_t row_g = static_cast<size_t>(ti.e) * p.w_rows + ti.mb * kBM + r;
#pragma unroll
            for (int a = 0; a < C::kNumA; ++a) {
                const size_t row = row_g + static_cast<size_t>(a) * p.m_out;
                if (row < srows) n_srow[a] = p.w_scales + row * kgroups;
            }
        };
        auto fetch = [&](uint16_t (&sb)[2]) {
            const int grp = n_ks * 2 + (g >> 1);           // the 128-K scale group of quarter g
#pragma unroll
            for (int a = 0; a < 2; ++a)
                sb[a] = (a < C::kNumA && n_srow[a] && grp < kgroups) ? __ldg(n_srow[a] + grp) : 0;
        };
        // scales of the stage being decoded (sb_cur), and of the next one
        // (sb_next): fetches run two stages ahead of their use
        set_rows();
        uint16_t sb_cur[2], sb_next[2];
        fetch(sb_cur);
        auto step = [&]() {
            if (++n_ks == KS) {
                n_ks = 0;
                n_tile += gridDim.x;
                set_rows();
            }
        };
        int c_tile = n_tile;          // tile of the stage being decoded
        step();
        fetch(sb_next);
        int stage = 0;
        uint32_t sphase = 0;
        int t = grp_id % C::kTmemAStages;
        uint32_t tphase = (grp_id / C::kTmemAStages) & 1;
        const int ch0 = ((2 * g) ^ (r & 7)) << 4, ch1 = ((2 * g + 1) ^ (r & 7)) << 4;
        while (c_tile < total_tiles) {
            const uint16_t sb0 = sb_cur[0], sb1 = sb_cur[1];
            sb_cur[0] = sb_next[0];
            sb_cur[1] = sb_next[1];
            c_tile = n_tile;
            step();
            fetch(sb_next);
            bool ok = mbar_wait(&full_bar[stage], sphase, abort_flag, p.err, 0);
            if (ok) ok = mbar_wait(&tfree_bar[t], tphase ^ 1, abort_flag, p.err, 0);
            if (!ok) break;
            tc_fence_after_sync();
            const uint8_t *st = ring + stage * C::kStageBytes + r * 128;
#pragma unroll
            for (int a = 0; a < C::kNumA; ++a) {
                const uint4 p0 = *reinterpret_cast<const uint4 *>(st + a * kPackedTile + ch0);
                const uint4 p1 = *reinterpret_cast<const uint4 *>(st + a * kPackedTile + ch1);
                const uint32_t words[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
                const __nv_bfloat162 s2 = bf16_pair(a == 0 ? sb0 : sb1);
                uint32_t out[32];
#pragma unroll
                for (int i = 0; i < 8; ++i) dequant_word(words[i], s2, out + 4 * i);
                tmem_st_32x32b_x32(tmem_a0 + (static_cast<uint32_t>(q * 32) << 16) + t * C::kSlotCols + qcol + a * 32,
                                   out);
            }
            tmem_wait_st();
            tc_fence_before_sync();
            mbar_arrive(&tready_bar[t]);
            if (++stage == STAGES) { stage = 0; sphase ^= 1; }
            // this group's slot for the next stage is GROUPS ring slots further on
            t += GROUPS;
            while (t >= C::kTmemAStages) { t -= C::kTmemAStages; tphase ^= 1; }
        }
    }

    // every role is done: the next kernel may start its set-up now
    griddep_launch_dependents();
    __syncthreads();
    if (*abort_flag) {
        for (int i = 0; i < 1000; ++i) __nanosleep(1000);
    }
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

// ------------------------------------------------------------------ host side

template <int BN, int STAGES, bool SWIGLU, int KSUB = 1>
cudaError_t run_bf16(const GemmArgs &g, cudaStream_t s) {
    using C = Bf16Cfg<BN, STAGES, SWIGLU, KSUB>;
    CUtensorMap ta, tb;
    const uint64_t a_rows = static_cast<uint64_t>(g.E) * g.w_rows;
    bool ok = make_map(&ta, g.w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, g.K, a_rows, kBK, kBM,
                       CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_token_map(&tb, g, kBoxN);
    if (!ok) return cudaErrorInvalidValue;
    auto kern = grouped_gemm_kernel<BN, STAGES, SWIGLU, KSUB>;
    cudaError_t st = ensure_dynamic_smem(kern, C::kSmemBytes);
    if (st != cudaSuccess) return st;
    const int grid = grid_for(g, BN);
    if (grid <= 0) return cudaSuccess;
    return launch_pdl(kern, dim3(grid), dim3(C::kThreads), C::kSmemBytes, s, ta, tb, make_params(g, BN));
}

template <int BN, int STAGES, bool SWIGLU, int GROUPS>
cudaError_t run_int4(const GemmArgs &g, cudaStream_t s) {
    using C = Int4Cfg<BN, STAGES, SWIGLU, GROUPS>;
    CUtensorMap ta, tb;
    const uint64_t a_rows = static_cast<uint64_t>(g.E) * g.w_rows;
    // packed weights: 128 bytes (K = 256) per row and stage, 128-byte swizzle
    bool ok = make_map(&ta, g.w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, g.K / 2, a_rows, 128, kBM,
                       CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_token_map(&tb, g, kBoxN);
    if (!ok) return cudaErrorInvalidValue;
    auto kern = grouped_gemm_int4_kernel<BN, STAGES, SWIGLU, GROUPS>;
    cudaError_t st = ensure_dynamic_smem(kern, C::kSmemBytes);
    if (st != cudaSuccess) return st;
    const int grid = grid_for(g, BN);
    if (grid <= 0) return cudaSuccess;
    return launch_pdl(kern, dim3(grid), dim3(C::kThreads), C::kSmemBytes, s, ta, tb, make_params(g, BN));
}

template <bool SWIGLU>
cudaError_t dispatch_bf16(const GemmArgs &g, cudaStream_t s) {
    const double avg = static_cast<double>(g.P) / g.E;   // pairs per expert if the load were even
    if constexpr (SWIGLU) {
        if (avg <= 24) return run_bf16<32, 3, SWIGLU, 2>(g, s);          // 72 KB stages (two 64-K blocks)
        if (avg <= 48) return run_bf16<64, 5, SWIGLU>(g, s);
        return run_bf16<128, 4, SWIGLU>(g, s);
    } else {
        if (avg <= 24) return run_bf16<32, 5, SWIGLU, 2>(g, s);          // 40 KB stages (two 64-K blocks)
        if (avg <= 48) return run_bf16<64, 8, SWIGLU>(g, s);
        return run_bf16<128, 6, SWIGLU>(g, s);
    }
}

template <bool SWIGLU>
cudaError_t dispatch_int4(const GemmArgs &g, cudaStream_t s) {
    const double avg = static_cast<double>(g.P) / g.E;
    // Measured on a B200 at the W4A16 decode shape (7168 x 2048, 8 rows per
    // expert): gate/up runs 4% faster with the weights decoded into TMEM for
    // tcgen05 MMAs, down 15% faster decoded straight into warp-level MMA
    // fragments (gemm_int4_warp_sm100.cu).
    if constexpr (SWIGLU) {
        if (avg <= 24) return run_int4<32, 4, SWIGLU, 2>(g, s);      // 48 KB stages, 3 slots of 128 K
        return run_int4<64, 3, SWIGLU, 4>(g, s);                     // 64 KB stages
    } else {
        if (avg <= 24) return launch_grouped_gemm_int4_warp(g, s);
        return run_int4<64, 4, SWIGLU, 2>(g, s);                     // 48 KB stages
    }
}

// Standalone W4A16 decoding: the same dequant_word as the GEMMs' decode warps.
__global__ void dequant_int4_kernel(const uint4 *__restrict__ q, const uint16_t *__restrict__ scales, int rows,
                                    int K, uint4 *__restrict__ out) {
    griddep_wait();
    const long long chunks_per_row = K / 32;   // 16 packed bytes = 32 values
    const long long total = static_cast<long long>(rows) * chunks_per_row;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long r = i / chunks_per_row;
        const int c = static_cast<int>(i - r * chunks_per_row);
        const __nv_bfloat162 s2 = bf16_pair(__ldg(scales + r * (K / 128) + (c * 32) / 128));
        const uint4 pk = __ldg(q + i);
        const uint32_t words[4] = {pk.x, pk.y, pk.z, pk.w};
        uint32_t o[16];
#pragma unroll
        for (int w = 0; w < 4; ++w) dequant_word(words[w], s2, o + 4 * w);
#pragma unroll
        for (int j = 0; j < 4; ++j) out[i * 4 + j] = make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
    }
}

// Many rows per expert: bf16 weights go to the tokens-on-M kernel.
bool uses_prefill_kernel(long long P, int E, int fmt) { return fmt == 0 && P >= 64LL * E; }

}  // namespace

bool gemm_gathers_in_kernel(int P, int E, int fmt) { return !uses_prefill_kernel(P, E, fmt); }

cudaError_t launch_grouped_gemm(const GemmArgs &g, cudaStream_t s) {
    if (g.P == 0) return cudaSuccess;
    if (g.fmt >= 2) return cudaErrorInvalidValue;      // MX formats: launch_grouped_gemm_mxfp8
    if (g.fmt == 0) {
        // many tokens per expert: weights on M across CTA pairs (gemm_wm_pair_sm100.cu)
        if (uses_prefill_kernel(g.P, g.E, g.fmt)) return launch_grouped_gemm_prefill(g, s);
        return g.swiglu ? dispatch_bf16<true>(g, s) : dispatch_bf16<false>(g, s);
    }
    return g.swiglu ? dispatch_int4<true>(g, s) : dispatch_int4<false>(g, s);
}

cudaError_t launch_dequant_int4(const uint8_t *q, const uint16_t *scales, int rows, int K, uint16_t *out,
                                cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    const long long total = static_cast<long long>(rows) * (K / 32);
    long long blocks = (total + 255) / 256;
    if (blocks > 148LL * 16) blocks = 148LL * 16;
    return launch_pdl(dequant_int4_kernel, dim3(static_cast<int>(blocks)), dim3(256), 0, s,
                      reinterpret_cast<const uint4 *>(q), scales, rows, K, reinterpret_cast<uint4 *>(out));
}

}  // namespace moe
