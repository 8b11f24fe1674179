// gemm_wm_pair_sm100.cu -- grouped GEMMs for many tokens per expert (bf16):
// weights on the MMA's M side across a CTA pair, tokens on the N side with
// the instruction N set per tile from the expert's routed-token count.
//
// Same results as the other grouped GEMMs (InfiniLM PR #500 Qwen3-MoE report,
// §2.2 step 2: gate/up with SwiGLU, then down, over every expert's slab of
// permuted rows). The operand roles follow the FlashInfer PR #7196 analysis,
// §2 (the 2-CTA M256 form with runtime MMA N):
//  - A tile = 256 weight rows, split across the two CTAs of a cluster
//    (128 rows each); one tcgen05.mma.cta_group::2 per K step, M = 256.
//  - B tile = up to 256 token rows of one expert; the instruction N is the
//    tile's token count rounded up to 16, so an expert's last tile costs the
//    rows it has, not a whole 256-row block.
//  - The pair's MMA reads B rows [0, N/2) from the leading CTA's shared
//    memory and rows [N/2, N) from the other CTA's, at the same offset. So
//    the non-leading CTA loads its token rows starting N/2 rows into the
//    tile: a shift that follows the runtime N, not the fixed block size.
//  - gate/up: CTA r holds the gate rows of features fb*128 + 64r + [0, 64) in
//    its A rows 0-63 and the up rows of the same features in A rows 64-127.
//    The accumulator lanes of g and u of one feature are then 64 apart in
//    the same CTA's TMEM; the warp reading gate lanes and the warp reading
//    the matching up lanes swap halves of each 32-token chunk through shared
//    memory, and each forms act = bf16(silu(g) u) for its 16 tokens.
//  - down: CTA r holds output features fb*256 + 128r + [0, 128).
//  - Epilogue threads own one feature each; a warp stores 32 consecutive
//    features (64 bytes) of each token row.
// Warp roles: warp 0 TMA (both CTAs), warp 1 MMA (leading CTA) and TMEM
// owner, warps 2-9 epilogue over a double-buffered 2 x 256-column fp32
// accumulator: two sets of 4 warps split a tile's columns, each warp loads the
// next 32 columns while it stores the current ones and hands the buffer back
// right after its last tcgen05.ld of the tile.
// Every mbarrier wait is bounded; the named-barrier hand-off between epilogue
// warps is entered only after a bounded wait succeeded, and both warps of a
// pair take the same number of steps.
#include "gemm_common.cuh"
#include "launch_util.cuh"

namespace moe {
namespace {

using namespace gemm;

constexpr int kPairM = 256;                          // weight rows per pair tile (MMA M)
constexpr int kTokBlock = 256;                       // token rows per tile at most (MMA N)
constexpr int kABox = 64;                            // weight rows per TMA box (gate/up: gate and up halves)
constexpr int kBBox = 128;                           // token rows per TMA box: one box per stage
constexpr int kTileA = 128 * kBK * 2;                // 16 KB: this CTA's 128 weight rows
constexpr int kTileB = (kTokBlock / 2) * kBK * 2;    // 16 KB: up to 128 token rows of this CTA
constexpr int kBBoxBytes = kBBox * kBK * 2;          // 16 KB
constexpr int kStage = kTileA + kTileB;              // 32 KB
constexpr int kAccCols = kTokBlock;                  // fp32 accumulator columns per buffer
constexpr int kPairXchgBytes = 2 * 2 * 16 * 32 * 4;  // one warp pair's gate/up hand-off: 2 buffers x 2 x 16 x 32 fp32

// 8 epilogue warps: two sets of 4 (one per TMEM lane quarter), each set
// covering half of a tile's 32-column chunks, so that a tile's accumulator is
// read and handed back in half the time; for gate/up the 8 form 4 gate/up
// warp pairs.
template <bool SWIGLU, int STAGES>
struct WmPairCfg {
    static constexpr int kEpiWarps = 8;
    static constexpr int kThreads = 64 + 32 * kEpiWarps;
    static constexpr int kXchgBytes = SWIGLU ? 4 * kPairXchgBytes : 0;
    static constexpr int kRingBytes = STAGES * kStage;
    static constexpr int kNumBars = 2 * STAGES + 2 + 2 + 1;
    static constexpr int kSmemBytes =
        1024 + kRingBytes + kXchgBytes + 8 * kNumBars + 64 + 2 * (kMaxExperts + 1) * 4;
    static_assert(kSmemBytes + 64 <= kSmemLimit, "shared memory");
};

// Named barriers of the gate/up epilogue (barrier 0 is __syncthreads): per
// warp pair pq (0-3), "go" carries the gate warp's decision for the tile,
// "xchg" separates the writes and reads of one chunk's hand-off buffer.
__device__ __forceinline__ int bar_go(int pq) { return 1 + pq; }
__device__ __forceinline__ int bar_xchg(int pq) { return 5 + pq; }

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ uint16_t bf16_rn_bits(float v) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

template <bool SWIGLU, int STAGES>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(320, 1)
grouped_gemm_wm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                            const Params p) {
    using C = WmPairCfg<SWIGLU, STAGES>;
    constexpr int kFeatPerTile = SWIGLU ? 128 : 256;         // output features per pair tile
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *ring = smem;                                    // STAGES x [A own 128 rows | B own rows]
    float *xchg = reinterpret_cast<float *>(ring + C::kRingBytes);   // gate/up hand-off buffers
    uint64_t *bars = reinterpret_cast<uint64_t *>(ring + C::kRingBytes + C::kXchgBytes);
    uint64_t *full_bar = bars;                               // used in the leading CTA: both CTAs' bytes
    uint64_t *empty_bar = full_bar + STAGES;                 // each CTA's own (MMA commit to both)
    uint64_t *tfull_bar = empty_bar + STAGES;                // each CTA's own (MMA commit to both)
    uint64_t *tempty_bar = tfull_bar + 2;                    // used in the leading CTA: 8 warp arrivals
    uint64_t *drain_bar = tempty_bar + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain_bar + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
    volatile int *go_flag = reinterpret_cast<volatile int *>(tmem_holder + 2);     // [4]
    int *off_s = reinterpret_cast<int *>(tmem_holder + 16);
    int *pre_s = off_s + (kMaxExperts + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int rank = static_cast<int>(cluster_ctarank());   // 0 = leading CTA of the pair
    const int E = p.E;
    const int MB = (p.m_out + kFeatPerTile - 1) / kFeatPerTile;     // feature blocks
    const int KB = (p.K + kBK - 1) / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull_bar[b], 1);
            mbar_init(&tempty_bar[b], 2 * C::kEpiWarps);      // every epilogue warp of both CTAs
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
        tmem_alloc_pair(tmem_holder, 2 * kAccCols);
        tmem_relinquish_pair();
    }
    // With kGemmHintOffsetsReady, offsets were complete before the previous
    // kernel started: the tile list and the weight tiles of the first ring
    // stages need not wait for it (only the token rows do).
    const bool early = (p.hints & kGemmHintOffsetsReady) != 0;
    if (!early) griddep_wait();
    build_tile_prefix<C::kThreads>(p.offsets, E, MB, kTokBlock, off_s, pre_s, p.P, p.err);
    tc_fence_before_sync();
    __syncthreads();
    cluster_sync();                                          // barriers of both CTAs initialised
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_holder;
    const int total_tiles = pre_s[E];
    const int first_tile = static_cast<int>(cluster_id_x());
    const int tile_step = static_cast<int>(cluster_count_x());

    if (warp == 0) {
        // ============================ TMA producer (both CTAs) ==================
        if (lane == 0) {
            const uint64_t pol_w = l2_policy_evict_last();
            const uint64_t pol_x = l2_policy_evict_last();
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            // the A rows of this CTA for a tile: two 64-row boxes
            auto a_rows = [&](const TileInfo &ti, int &r0, int &r1) {
                if (SWIGLU) {
                    r0 = ti.e * p.w_rows + ti.mb * 128 + 64 * rank;     // gate rows
                    r1 = r0 + p.m_out;                                  // the matching up rows
                } else {
                    r0 = ti.e * p.w_rows + ti.mb * 256 + 128 * rank;   // one 128-row box
                    r1 = -1;
                }
            };
            int preloaded = 0;
            if (early) {
                for (int tile = first_tile; tile < total_tiles && preloaded < STAGES; tile += tile_step) {
                    const TileInfo ti = decode_tile(tile, pre_s, off_s, E, MB, kTokBlock);
                    const int nbox = (ti.n_mma / 2 + kBBox - 1) / kBBox;
                    const uint32_t tx = 2u * (kTileA + nbox * kBBoxBytes);
                    int r0, r1;
                    a_rows(ti, r0, r1);
                    for (int kb = 0; kb < KB && preloaded < STAGES; ++kb, ++preloaded) {
                        const uint32_t full_leader = cluster_map(smem_u32(&full_bar[preloaded]), 0);
                        if (rank == 0) mbar_arrive_expect_tx(&full_bar[preloaded], tx);
                        uint8_t *st = ring + preloaded * kStage;
                        tma_load_2d_pair(st, &tmA, full_leader, kb * kBK, r0, pol_w);
                        if (SWIGLU) tma_load_2d_pair(st + kTileA / 2, &tmA, full_leader, kb * kBK, r1, pol_w);
                    }
                }
                griddep_wait();
            }
            int it = 0;
            for (int tile = first_tile; tile < total_tiles && ok; tile += tile_step) {
                const TileInfo ti = decode_tile(tile, pre_s, off_s, E, MB, kTokBlock);
                const int half = ti.n_mma / 2;                       // token rows from each CTA
                const int nbox = (half + kBBox - 1) / kBBox;
                const uint32_t tx = 2u * (kTileA + nbox * kBBoxBytes);
                const int b_row = ti.row0 + rank * half;             // the non-leading CTA's shift
                int r0, r1;
                a_rows(ti, r0, r1);
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    ok = mbar_wait(&empty_bar[stage], phase ^ 1, abort_flag, p.err, 128);
                    if (!ok) break;
                    const uint32_t full_leader = cluster_map(smem_u32(&full_bar[stage]), 0);
                    uint8_t *st = ring + stage * kStage;
                    if (it >= preloaded) {
                        if (rank == 0) mbar_arrive_expect_tx(&full_bar[stage], tx);
                        tma_load_2d_pair(st, &tmA, full_leader, kb * kBK, r0, pol_w);
                        if (SWIGLU) tma_load_2d_pair(st + kTileA / 2, &tmA, full_leader, kb * kBK, r1, pol_w);
                    }
                    for (int b = 0; b < nbox; ++b)
                        tma_load_2d_pair(st + kTileA + b * kBBoxBytes, &tmB, full_leader, kb * kBK,
                                         b_row + b * kBBox, pol_x);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
            }
        }
    } else if (warp == 1) {
        // ============================ MMA issuer (leading CTA) ==================
        if (early) griddep_wait();
        if (lane == 0 && rank == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int buf = 0;
            uint32_t bphase = 0;
            bool ok = true;
            for (int tile = first_tile; tile < total_tiles && ok; tile += tile_step) {
                const TileInfo ti = decode_tile(tile, pre_s, off_s, E, MB, kTokBlock);
                const uint32_t idesc = idesc_bf16_f32(kPairM, ti.n_mma);
                ok = mbar_wait(&tempty_bar[buf], bphase ^ 1, abort_flag, p.err);
                if (!ok) break;
                tc_fence_after_sync();
                const uint32_t d = tmem_base + buf * kAccCols;
                for (int kb = 0; kb < KB; ++kb) {
                    ok = mbar_wait(&full_bar[stage], phase, abort_flag, p.err, 0);
                    if (!ok) break;
                    tc_fence_after_sync();
                    const uint32_t st = smem_u32(ring + stage * kStage);
                    const uint64_t da = sw128_kmajor_desc(st);
                    const uint64_t db = sw128_kmajor_desc(st + kTileA);
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k)
                        umma_bf16_ss_pair(d, da + 2 * k, db + 2 * k, idesc, (kb | k) != 0);
                    umma_commit_pair(&empty_bar[stage], 0x3);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                umma_commit_pair(&tfull_bar[buf], 0x3);
                if (++buf == 2) { buf = 0; bphase ^= 1; }
            }
            umma_commit_pair(drain_bar, 0x1);
            volatile int never = 0;
            mbar_wait(drain_bar, 0, &never, p.err);
        }
    } else {
        // ====================== warps 2+: epilogue (both CTAs) ==================
        if (early) griddep_wait();
        const int q = warp & 3;                              // TMEM lane quarter of this warp
        const uint32_t tempty_leader0 = cluster_map(smem_u32(&tempty_bar[0]), 0);
        const uint32_t tempty_leader1 = cluster_map(smem_u32(&tempty_bar[1]), 0);
        int buf = 0;
        uint32_t bphase = 0;
        // TMEM accumulator buffer handed back to the MMA issuer once this
        // warp's last tcgen05.ld of the tile has completed (every lane has
        // passed tcgen05.wait::ld). The arrive orders only those completed
        // loads, so it is relaxed: a release would first wait for the warp's
        // outstanding global stores.
        auto release = [&]() {
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster_relaxed(buf ? tempty_leader1 : tempty_leader0);
        };
        if (!SWIGLU) {
            // warps 2-5 store the first half of a tile's 32-column chunks,
            // warps 6-9 the second half, each warp its 32 features
            const int h = (warp - 2) >> 2;
            const int f_in_tile = 128 * rank + 32 * q + lane;
            for (int tile = first_tile; tile < total_tiles; tile += tile_step) {
                const TileInfo ti = decode_tile(tile, pre_s, off_s, E, MB, kTokBlock);
                if (!__shfl_sync(0xffffffffu, mbar_wait(&tfull_bar[buf], bphase, abort_flag, p.err, 512), 0)) break;
                tc_fence_after_sync();
                const int nch = (ti.valid + 31) >> 5;
                const int split = (nch + 1) >> 1;
                const int c_lo = h ? split : 0, c_hi = h ? nch : split;
                if (c_lo >= c_hi) {
                    release();
                    if (++buf == 2) { buf = 0; bphase ^= 1; }
                    continue;
                }
                const int f = ti.mb * kFeatPerTile + f_in_tile;
                const bool f_ok = f < p.m_out;
                const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * kAccCols;
                uint16_t *col = p.out + static_cast<size_t>(ti.row0) * p.m_out + f;
                const size_t row_stride = static_cast<size_t>(p.m_out);
                auto store = [&](const uint32_t (&v)[32], int c0) {
                    if (!f_ok) return;
                    uint16_t *dst = col + static_cast<size_t>(c0) * row_stride;
                    const int n = min(32, ti.valid - c0);
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        if (j < n) *dst = bf16_rn_bits(__uint_as_float(v[j]));
                        dst += row_stride;
                    }
                };
                // two register sets: the next 32 columns load while this set is stored
                const int c_end = 32 * c_hi;
                uint32_t va[32], vb[32];
                tmem_ld_32x32b_x32(tb + 32 * c_lo, va);
                tmem_wait_ld();
                for (int c0 = 32 * c_lo;; c0 += 64) {
                    const bool more_a = c0 + 32 < c_end;
                    if (more_a) tmem_ld_32x32b_x32(tb + c0 + 32, vb); else release();
                    store(va, c0);
                    if (!more_a) break;
                    tmem_wait_ld();
                    const bool more_b = c0 + 64 < c_end;
                    if (more_b) tmem_ld_32x32b_x32(tb + c0 + 64, va); else release();
                    store(vb, c0 + 32);
                    if (!more_b) break;
                    tmem_wait_ld();
                }
                if (++buf == 2) { buf = 0; bphase ^= 1; }
            }
        } else {
            // Warp pair (gate warp q < 2, up warp q + 2, same column half h)
            // shares 32 features of each 32-token chunk of its half of the
            // tile: the gate warp hands g of tokens 16-31 to the up warp, the
            // up warp hands u of tokens 0-15 to the gate warp, and each forms
            // act for its 16 tokens. Two hand-off buffers alternate, so one
            // barrier per chunk orders every write after the partner's read
            // of the same buffer two chunks earlier.
            const int h = (warp - 2) >> 2;                   // column half: warps 2-5 first, 6-9 second
            const bool gate_warp = q < 2;
            const int pq = (q & 1) + 2 * h;                  // warp pair index
            float *xb = xchg + pq * (kPairXchgBytes / 4);    // [buffer][giver: gate, up][16 tokens][32 lanes]
            const int f_in_tile = 64 * rank + 32 * (q & 1) + lane;
            uint32_t xbuf = 0;
            for (int tile = first_tile; tile < total_tiles; tile += tile_step) {
                const TileInfo ti = decode_tile(tile, pre_s, off_s, E, MB, kTokBlock);
                const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * kAccCols;
                if (gate_warp) {
                    // one decision for the pair (the barriers below are collective)
                    const bool ok =
                        __shfl_sync(0xffffffffu, mbar_wait(&tfull_bar[buf], bphase, abort_flag, p.err, 512), 0);
                    if (lane == 0) go_flag[pq] = ok ? 1 : 0;
                }
                named_bar_sync(bar_go(pq), 64);
                if (!go_flag[pq]) break;
                // the phase has completed (the gate warp saw it): this returns at
                // once and orders this warp's TMEM reads after the MMAs
                if (!gate_warp) mbar_wait(&tfull_bar[buf], bphase, abort_flag, p.err, 512);
                tc_fence_after_sync();
                // this half's columns: chunks [c_lo, c_hi) of 32
                const int nch = (ti.valid + 31) >> 5;
                const int split = (nch + 1) >> 1;
                const int c_lo = h ? split : 0, c_hi = h ? nch : split;
                if (c_lo >= c_hi) {
                    release();
                    if (++buf == 2) { buf = 0; bphase ^= 1; }
                    continue;
                }
                const int f = ti.mb * kFeatPerTile + f_in_tile;
                const bool f_ok = f < p.m_out;
                // this warp's 16 tokens of each chunk: 0-15 (gate warp) or 16-31 (up warp)
                const int my_half = gate_warp ? 0 : 16;
                uint16_t *col = p.out + static_cast<size_t>(ti.row0 + my_half) * p.m_out + f;
                auto chunk = [&](const uint32_t (&v)[32], int c0) {
                    float *give = xb + xbuf * (2 * 16 * 32) + (gate_warp ? 0 : 16 * 32);
                    const float *take = xb + xbuf * (2 * 16 * 32) + (gate_warp ? 16 * 32 : 0);
#pragma unroll
                    for (int j = 0; j < 16; ++j) give[j * 32 + lane] = __uint_as_float(gate_warp ? v[16 + j] : v[j]);
                    named_bar_sync(bar_xchg(pq), 64);
                    if (f_ok) {
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int t = c0 + my_half + j;
                            if (t < ti.valid) {
                                const float other = take[j * 32 + lane];
                                const float gv = gate_warp ? __uint_as_float(v[j]) : other;
                                const float uv = gate_warp ? other : __uint_as_float(v[16 + j]);
                                const float a = gv / (1.0f + expf(-gv)) * uv;
                                col[static_cast<size_t>(c0 + j) * p.m_out] = bf16_rn_bits(a);
                            }
                        }
                    }
                    xbuf ^= 1;
                };
                const int c_end = 32 * c_hi;
                uint32_t va[32], vb[32];
                tmem_ld_32x32b_x32(tb + 32 * c_lo, va);
                tmem_wait_ld();
                for (int c0 = 32 * c_lo;; c0 += 64) {
                    const bool more_a = c0 + 32 < c_end;
                    if (more_a) tmem_ld_32x32b_x32(tb + c0 + 32, vb); else release();
                    chunk(va, c0);
                    if (!more_a) break;
                    tmem_wait_ld();
                    const bool more_b = c0 + 64 < c_end;
                    if (more_b) tmem_ld_32x32b_x32(tb + c0 + 64, va); else release();
                    chunk(vb, c0 + 32);
                    if (!more_b) break;
                    tmem_wait_ld();
                }
                if (++buf == 2) { buf = 0; bphase ^= 1; }
            }
        }
    }

    // every role is done: the next kernel may start its set-up now
    griddep_launch_dependents();
    __syncthreads();
    if (*abort_flag) {
        for (int i = 0; i < 1000; ++i) __nanosleep(1000);
    }
    cluster_sync();                                          // no remote arrival or MMA left in flight
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc_pair(tmem_base, 2 * kAccCols);
    }
}

template <bool SWIGLU>
cudaError_t run_wm_pair(const GemmArgs &g, cudaStream_t s) {
    constexpr int STAGES = SWIGLU ? 5 : 6;
    using C = WmPairCfg<SWIGLU, STAGES>;
    CUtensorMap ta, tb;
    const uint64_t a_rows = static_cast<uint64_t>(g.E) * g.w_rows;
    bool ok = make_map(&ta, g.w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, g.K, a_rows, kBK, SWIGLU ? kABox : 128,
                       CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_map(&tb, g.a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, g.K, static_cast<uint64_t>(g.P), kBK, kBBox,
                       CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok || g.perm) return cudaErrorInvalidValue;
    auto kern = grouped_gemm_wm_pair_kernel<SWIGLU, STAGES>;
    cudaError_t st = ensure_dynamic_smem(kern, C::kSmemBytes);
    if (st != cudaSuccess) return st;
    constexpr int kFeat = SWIGLU ? 128 : 256;
    const long long MB = (g.m_out + kFeat - 1) / kFeat;
    const long long max_tiles =
        ((static_cast<long long>(g.P) + kTokBlock - 1) / kTokBlock + std::min(g.E, g.P)) * MB;
    const int pairs = static_cast<int>(std::min<long long>(num_sms() / 2, max_tiles));
    if (pairs <= 0) return cudaSuccess;
    Params p = make_params(g, kTokBlock);
    p.evict_first_weights = 0;
    return launch_pdl(kern, dim3(2 * pairs), dim3(C::kThreads), C::kSmemBytes, s, ta, tb, p);
}

}  // namespace

cudaError_t launch_grouped_gemm_wm_pair(const GemmArgs &g, cudaStream_t s) {
    if (g.P == 0) return cudaSuccess;
    return g.swiglu ? run_wm_pair<true>(g, s) : run_wm_pair<false>(g, s);
}

}  // namespace moe
