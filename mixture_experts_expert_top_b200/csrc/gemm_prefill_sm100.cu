// gemm_prefill_sm100.cu -- grouped GEMMs for many tokens per expert (bf16)
// whose token rows are read through perm (TMA gather4) rather than from a
// permuted copy; permuted copies go to gemm_wm_pair_sm100.cu.
//
// Same results as the kernels of gemm_sm100.cu (InfiniLM PR #500 Qwen3-MoE
// report, §2.2 step 2: gate/up with SwiGLU, then down, over every expert's
// slab of permuted rows), with the operands the other way round: tokens are
// the MMA's A operand (M = 128 token rows per tile) and weights the B operand
// (N = 256 weight rows per tile).
//  - gate/up: the 256 B rows are 128 gate rows and the matching 128 up rows,
//    so one 128 x 256 MMA per K step accumulates g in TMEM columns 0-127 and
//    u in columns 128-255 of the same lane; the epilogue thread that owns a
//    token row computes act = bf16(silu(g) * u) for 128 features.
//  - down: the 256 B rows are 256 output features.
//  - Each epilogue thread owns one token row, so its stores are contiguous
//    16-byte vectors of that row.
//  - Tiles are (expert, 128-token block, feature block); the token block of
//    an expert's last tile may run past its rows: those accumulator rows are
//    computed but never stored.
// Warp roles as in gemm_sm100.cu: warp 0 TMA, warp 1 MMA + TMEM owner,
// warps 2-5 epilogue over a double-buffered 2 x 256-column accumulator.
#include "gemm_common.cuh"
#include "launch_util.cuh"

namespace moe {
namespace {

using namespace gemm;

constexpr int kTokM = 128;                          // token rows per tile (MMA M)
constexpr int kRowsB = 256;                         // weight rows per tile (MMA N)
constexpr int kTileA = kTokM * kBK * 2;             // 16 KB
constexpr int kTileB = kRowsB * kBK * 2;            // 32 KB
constexpr int kStageBytes = kTileA + kTileB;        // 48 KB
constexpr int kAccCols = kRowsB;                    // fp32 accumulator columns per buffer

// Reads this thread's accumulator row (kFeat output features) from TMEM and
// packs it to bf16 pairs: SwiGLU over columns c (gate) and 128 + c (up), or
// the plain row for down. Nothing is stored yet, so the caller can hand the
// TMEM buffer back before its global stores.
template <bool SWIGLU>
__device__ __forceinline__ void load_acc_row(uint32_t tb, uint32_t (&packed)[(SWIGLU ? 128 : 256) / 2]) {
    constexpr int kFeat = SWIGLU ? 128 : 256;
#pragma unroll
    for (int c = 0; c < kFeat; c += 32) {
        uint32_t g[32];
        tmem_ld_32x32b_x32(tb + c, g);
        if (SWIGLU) {
            uint32_t u[32];
            tmem_ld_32x32b_x32(tb + 128 + c, u);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                float a[2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float gv = __uint_as_float(g[2 * j + h]);
                    a[h] = gv / (1.0f + expf(-gv)) * __uint_as_float(u[2 * j + h]);
                }
                const __nv_bfloat162 v = __floats2bfloat162_rn(a[0], a[1]);
                packed[c / 2 + j] = *reinterpret_cast<const uint32_t *>(&v);
            }
        } else {
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const __nv_bfloat162 v =
                    __floats2bfloat162_rn(__uint_as_float(g[2 * j]), __uint_as_float(g[2 * j + 1]));
                packed[c / 2 + j] = *reinterpret_cast<const uint32_t *>(&v);
            }
        }
    }
}

// Stores a packed bf16 row segment of kFeat features at orow[f0 ...], 16 bytes
// at a time, features past m_out dropped.
template <int NF>
__device__ __forceinline__ void store_row(uint16_t *orow, int f0, int m_out, const uint32_t (&packed)[NF / 2]) {
#pragma unroll
    for (int v = 0; v < NF / 8; ++v) {
        const int f = f0 + 8 * v;
        if (f < m_out)
            *reinterpret_cast<uint4 *>(orow + f) =
                make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
    }
}

template <int STAGES>
struct PrefillCfg {
    static constexpr int kRingBytes = STAGES * kStageBytes;
    static constexpr int kNumBars = 2 * STAGES + 2 + 2 + 1;
    static constexpr int kSmemBytes = 1024 + kRingBytes + 8 * kNumBars + 64 + 2 * (kMaxExperts + 1) * 4;
    static_assert(kSmemBytes + 64 <= kSmemLimit, "shared memory");
};

template <bool SWIGLU, int STAGES>
__global__ void __launch_bounds__(192, 1)
grouped_gemm_prefill_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                            const Params p) {
    using C = PrefillCfg<STAGES>;
    constexpr int kFeat = SWIGLU ? 128 : 256;       // output features per tile
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *ring = smem;                                    // STAGES x [A tokens | B weights]
    uint64_t *bars = reinterpret_cast<uint64_t *>(ring + C::kRingBytes);
    uint64_t *full_bar = bars;
    uint64_t *empty_bar = full_bar + STAGES;
    uint64_t *tfull_bar = empty_bar + STAGES;
    uint64_t *tempty_bar = tfull_bar + 2;
    uint64_t *drain_bar = tempty_bar + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain_bar + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
    int *off_s = reinterpret_cast<int *>(tmem_holder + 16);
    int *pre_s = off_s + (kMaxExperts + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int E = p.E;
    const int NB = (p.m_out + kFeat - 1) / kFeat;            // feature blocks
    const int KB = (p.K + kBK - 1) / kBK;

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
        tmem_alloc(tmem_holder, 2 * kAccCols);
        tmem_relinquish();
    }
    // tiles of expert e: ceil(rows / 128) token blocks x NB feature blocks
    // barriers, tensor maps and TMEM are set up while the previous kernel drains
    griddep_wait();
    build_tile_prefix<192>(p.offsets, E, NB, kTokM, off_s, pre_s, p.P, p.err);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_holder;
    const int total_tiles = pre_s[E];

    if (warp == 0) {
        // ================================ TMA producer ==========================
        // Lane 0 runs the ring; with perm, all 32 lanes issue the token rows as
        // gather4 loads (lane i: tile rows 4i .. 4i+3) straight from hidden.
        const uint64_t pol = l2_policy_evict_last();
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
            // decode_tile: .mb = feature block, .row0/.valid = token block
            const TileInfo ti = decode_tile(tile, pre_s, off_s, E, NB, kTokM);
            const int f0 = ti.mb * kFeat;
            const int b_row0 = ti.e * p.w_rows + f0;
            const int b_row1 = SWIGLU ? b_row0 + p.m_out : b_row0 + 128;
            int tr[4] = {0, 0, 0, 0};
            if (p.perm) {
#pragma unroll
                for (int j = 0; j < 4; ++j) tr[j] = token_row(p, ti.row0 + 4 * lane + j);
            }
            for (int kb = 0; kb < KB; ++kb) {
                if (lane == 0) ok = mbar_wait(&empty_bar[stage], phase ^ 1, abort_flag, p.err, 256);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                uint8_t *st = ring + stage * kStageBytes;
                if (lane == 0) mbar_arrive_expect_tx(&full_bar[stage], kStageBytes);
                __syncwarp();
                if (p.perm)
                    tma_gather4(st + lane * 4 * kBK * 2, &tmA, &full_bar[stage], kb * kBK, tr[0], tr[1], tr[2], tr[3],
                                pol);
                else if (lane == 0)
                    tma_load_2d(st, &tmA, &full_bar[stage], kb * kBK, ti.row0, pol);
                if (lane == 0) {
                    tma_load_2d(st + kTileA, &tmB, &full_bar[stage], kb * kBK, b_row0, pol);
                    tma_load_2d(st + kTileA + kTileB / 2, &tmB, &full_bar[stage], kb * kBK, b_row1, pol);
                }
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
        }
    } else if (warp == 1) {
        // ================================ MMA issuer ============================
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(kTokM, kRowsB);
            int stage = 0;
            uint32_t phase = 0;
            int buf = 0;
            uint32_t bphase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
                ok = mbar_wait(&tempty_bar[buf], bphase ^ 1, abort_flag, p.err);
                if (!ok) break;
                tc_fence_after_sync();
                const uint32_t d = tmem_base + buf * kAccCols;
                for (int kb = 0; kb < KB; ++kb) {
                    ok = mbar_wait(&full_bar[stage], phase, abort_flag, p.err, 0);
                    if (!ok) break;
                    tc_fence_after_sync();
                    const uint32_t st = smem_u32(ring + stage * kStageBytes);
                    const uint64_t da = sw128_kmajor_desc(st);
                    const uint64_t db = sw128_kmajor_desc(st + kTileA);
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k)
                        umma_bf16_ss(d, da + 2 * k, db + 2 * k, idesc, (kb | k) != 0);
                    umma_commit(&empty_bar[stage]);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                umma_commit(&tfull_bar[buf]);
                if (++buf == 2) { buf = 0; bphase ^= 1; }
            }
            umma_commit(drain_bar);
            volatile int never = 0;
            mbar_wait(drain_bar, 0, &never, p.err);
        }
    } else {
        // ============================ warps 2-5: epilogue ========================
        const int q = warp & 3;
        const int tr = q * 32 + lane;                       // token row of the tile owned by this thread
        int buf = 0;
        uint32_t bphase = 0;
        for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
            const TileInfo ti = decode_tile(tile, pre_s, off_s, E, NB, kTokM);
            if (!mbar_wait(&tfull_bar[buf], bphase, abort_flag, p.err, 512)) break;
            tc_fence_after_sync();
            const int f0 = ti.mb * kFeat;
            const bool row_ok = tr < ti.valid;
            uint16_t *orow = p.out + static_cast<size_t>(ti.row0 + (row_ok ? tr : 0)) * p.m_out;
            const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * kAccCols;
            uint32_t packed[kFeat / 2];
            load_acc_row<SWIGLU>(tb, packed);
            tc_fence_before_sync();
            mbar_arrive(&tempty_bar[buf]);          // buffer free before the stores go out
            if (row_ok) store_row<kFeat>(orow, f0, p.m_out, packed);
            if (++buf == 2) { buf = 0; bphase ^= 1; }
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
        tmem_dealloc(tmem_base, 2 * kAccCols);
    }
}

template <bool SWIGLU>
cudaError_t run_prefill(const GemmArgs &g, cudaStream_t s) {
    constexpr int STAGES = 4;
    using C = PrefillCfg<STAGES>;
    CUtensorMap ta, tb;
    const uint64_t b_rows = static_cast<uint64_t>(g.E) * g.w_rows;
    bool ok = make_token_map(&ta, g, kTokM) &&
              make_map(&tb, g.w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, g.K, b_rows, kBK, 128,
                       CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok) return cudaErrorInvalidValue;
    auto kern = grouped_gemm_prefill_kernel<SWIGLU, STAGES>;
    cudaError_t st = ensure_dynamic_smem(kern, C::kSmemBytes);
    if (st != cudaSuccess) return st;
    constexpr int kFeat = SWIGLU ? 128 : 256;
    const long long NB = (g.m_out + kFeat - 1) / kFeat;
    const long long max_tiles = ((static_cast<long long>(g.P) + kTokM - 1) / kTokM + std::min(g.E, g.P)) * NB;
    const int grid = static_cast<int>(std::min<long long>(num_sms(), max_tiles));
    if (grid <= 0) return cudaSuccess;
    Params p = make_params(g, kTokM);
    return launch_pdl(kern, dim3(grid), dim3(192), C::kSmemBytes, s, ta, tb, p);
}

}  // namespace

cudaError_t launch_grouped_gemm_prefill(const GemmArgs &g, cudaStream_t s) {
    if (g.P == 0) return cudaSuccess;
    // rows already permuted: weights on M across CTA pairs, runtime token N
    // (gemm_wm_pair_sm100.cu); rows read through perm: this file's kernel
    if (!g.perm) return launch_grouped_gemm_wm_pair(g, s);
    return g.swiglu ? run_prefill<true>(g, s) : run_prefill<false>(g, s);
}

}  // namespace moe
