// gemm_mxfp8_sm100.cu -- the MoE layer's grouped GEMMs with MXFP8 weights on
// sm_100a's block-scaled tensor-core MMA (tcgen05.mma kind::mxf8f6f4 with
// E8M0 block scales), and the MX quantisation of the activations they take.
//
// Format (OCP Microscaling Formats (MX) v1.0): E4M3 elements, one E8M0 scale
// 2^(c-127) per 32 consecutive K elements of a row. The GC-MoE abstract runs
// its expert GEMMs in FP8 / FP4; the block-scaled MMA takes both operands in
// MX form, so the activations are MX-quantised by the layer: hidden before
// gate/up (mx_quantize_kernel) and act, after its bf16 rounding, before down
// (in the gate/up epilogue). Quantisation of a block of 32: e = floor(log2
// max|x|) - 8 clamped to [-127, 127] (-127 for an all-zero block), elements
// x * 2^-e (exact in fp32) converted to E4M3 with round-to-nearest-even and
// saturation to +-448.
//
// GEMM layout as in the bf16 weights-on-M kernel (gemm_sm100.cu): weights are
// operand A (M = 128 rows per tile), tokens operand B with N = the tile's
// rows rounded up to 16; gate/up tiles hold the gate and the matching up
// rows and accumulate g and u in two TMEM accumulators. A ring stage holds
// K = 128 (one 128-byte swizzled row per operand row), so one stage is four
// MMAs of K = 32 per accumulator. The stage's scale factors (128 weight rows
// x 4 K blocks, and the same for up to 128 token rows: 512 bytes each, row m
// at byte (m % 32) * 16 + (m / 32) * 4 + kb) are written to shared memory by
// the producer warp's lanes, copied into a TMEM slot of that stage with
// tcgen05.cp (32x128b, replicated to every lane quarter) by the MMA thread,
// and selected per MMA by the K block index in the address's top bits.
//
// MXFP4 weights (W4 = true): E2M1 elements packed two per byte in global
// memory, times MXFP8 tokens, on the same MMA kind (mixed f8f6f4 operand
// types). The weight tiles are loaded by TMA as 4-bit elements
// (CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B): every 16 elements (8 bytes) land
// in 16 bytes of shared memory, the layout the MMA reads for 4-bit operands,
// so a stage holds the same K = 128 per 128-byte row as for E4M3 while HBM
// carries half the bytes. Everything else (scale factors, epilogues) is the
// MXFP8 kernel's.
#include <cuda_fp8.h>

#include "gemm_common.cuh"
#include "launch_util.cuh"

namespace moe {
namespace {

using namespace gemm;

constexpr int kMxBK = 128;                      // K elements (bytes) per stage and operand row
constexpr int kMxTileA = kBM * kMxBK;           // 16 KB
constexpr int kSfBlock = 512;                   // scale factors of 128 rows x 4 K blocks

// E4M3 code of x (round to nearest even, saturate to +-448).
__device__ __forceinline__ uint8_t e4m3_rn_sat(float x) {
    return static_cast<uint8_t>(__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3));
}

// Block exponent of an MX block from the bits of its max |x| (a non-negative
// float): floor(log2 amax) - 8, clamped to [-127, 127]; -127 for amax = 0.
__device__ __forceinline__ int mx_block_exponent(uint32_t amax_bits) {
    if (amax_bits == 0) return -127;
    const int biased = static_cast<int>(amax_bits >> 23);       // 0 for a subnormal max
    return max(biased - 127 - 8, -127);
}

// 2^-e as an fp32 (normal for every e the exponent rule gives).
__device__ __forceinline__ float mx_inverse_scale(int e) { return __uint_as_float(static_cast<uint32_t>(127 - e) << 23); }

// MX quantisation of bf16 rows [rows, K] (K % 32 == 0): one thread per 8
// elements, 4 consecutive lanes per 32-element block. Whole warps step
// through the vectors together (lanes past the end only take part in the
// shuffles), so the 4 lanes of a block are always in one warp.
__global__ void __launch_bounds__(256)
mx_quantize_kernel(const uint4 *__restrict__ x, long long total_vecs, uint2 *__restrict__ q,
                   uint8_t *__restrict__ scales) {
    griddep_launch_dependents();
    griddep_wait();
    const int lane = threadIdx.x & 31;
    const long long warp0 = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) - lane;
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long base = warp0; base < total_vecs; base += stride) {
        const long long i = base + lane;
        const bool in = i < total_vecs;
        float f[8];
        uint32_t amax = 0;
        if (in) {
            const uint4 v = __ldg(x + i);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                f[j] = bf16_bits_to_float((w[j >> 1] >> ((j & 1) * 16)) & 0xFFFFu);
                amax = max(amax, __float_as_uint(fabsf(f[j])));
            }
        }
        amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        if (!in) continue;
        const int e = mx_block_exponent(amax);
        const float inv = mx_inverse_scale(e);
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) lo |= static_cast<uint32_t>(e4m3_rn_sat(__fmul_rn(f[j], inv))) << (8 * j);
#pragma unroll
        for (int j = 0; j < 4; ++j) hi |= static_cast<uint32_t>(e4m3_rn_sat(__fmul_rn(f[4 + j], inv))) << (8 * j);
        q[i] = make_uint2(lo, hi);
        if ((i & 3) == 0) scales[i >> 2] = static_cast<uint8_t>(e + 127);
    }
}

template <int BN, int STAGES, bool SWIGLU>
struct MxCfg {
    static constexpr int kNumA = SWIGLU ? 2 : 1;
    static constexpr int kThreads = 192;
    static constexpr int kABytes = kNumA * kMxTileA;
    static constexpr int kBBytes = BN * kMxBK;
    static constexpr int kSfBytes = (kNumA + 1) * kSfBlock;           // A blocks, then the B block
    static constexpr int kStageBytes = ((kABytes + kBBytes + kSfBytes + 1023) / 1024) * 1024;
    static constexpr int kAccCols = SWIGLU ? 2 * BN : BN;
    static constexpr int kSfCols = 4 * (kNumA + 1);                  // TMEM columns of one stage's scales
    static constexpr int kTmemUsed = 2 * kAccCols + STAGES * kSfCols;
    static constexpr int kTmemCols = kTmemUsed <= 32 ? 32 : kTmemUsed <= 64 ? 64 : kTmemUsed <= 128 ? 128
                                   : kTmemUsed <= 256 ? 256 : 512;
    static constexpr int kRingBytes = STAGES * kStageBytes;
    static constexpr int kNumBars = 2 * STAGES + 2 + 2 + 1;
    static constexpr int kSmemBytes = 1024 + kRingBytes + 8 * kNumBars + 64 + 2 * (kMaxExperts + 1) * 4;
    static_assert(kTmemUsed <= 512, "TMEM holds 512 32-bit columns");
    static_assert(BN % kBoxN == 0 && BN <= 128, "BN");
    static_assert(kSmemBytes + 64 <= kSmemLimit, "shared memory");
};

struct MxParams {
    Params p;
    const uint8_t *w_sf;        // [E * w_rows, K/32] E8M0
    const uint8_t *x_sf;        // token rows' E8M0 scales [rows, K/32]
    uint8_t *out_q;             // gate/up: act E4M3 [P, I]; down: unused
    uint8_t *out_sf;            // gate/up: act E8M0 [P, I/32]; down: unused
    int w_total_rows;           // E * w_rows
    int x_rows;                 // rows of the token tensor (T with perm, else P)
};

template <int BN, int STAGES, bool SWIGLU, bool W4>
__global__ void __launch_bounds__(192, 1)
grouped_gemm_mxfp8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                          const MxParams mp) {
    using C = MxCfg<BN, STAGES, SWIGLU>;
    const Params &p = mp.p;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *ring = smem;                                    // STAGES x [A | A up | B | scale factors]
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
    const int MB = (p.m_out + kBM - 1) / kBM;
    const int KB = p.K / kMxBK;                              // K % 128 == 0
    const int sf_row_bytes = p.K / 32;

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
    griddep_wait();
    build_tile_prefix<C::kThreads>(p.offsets, E, MB, BN, off_s, pre_s, p.P, p.err);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_holder;
    const int total_tiles = pre_s[E];

    if (warp == 0) {
        // ================================ producer ==============================
        // Lane 0 runs the ring and the TMA loads (with perm, lanes i < N/4 issue
        // the token rows as gather4 loads); every lane writes the scale factors
        // of 4 weight rows (and 4 token rows) into the stage's 512-byte blocks.
        const uint64_t pol_w = p.evict_first_weights ? l2_policy_evict_first() : l2_policy_evict_last();
        const uint64_t pol_x = l2_policy_evict_last();
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
            const TileInfo ti = decode_tile(tile, pre_s, off_s, E, MB, BN);
            const int nbox = ti.n_mma / kBoxN;
            const int a_row = ti.e * p.w_rows + ti.mb * kBM;
            // a 4-bit weight tile moves (and counts) 8 bytes per 16 elements
            const uint32_t tx = (W4 ? C::kABytes / 2 : C::kABytes) + nbox * kBoxN * kMxBK;
            const bool gather_lane = p.perm && 4 * lane < ti.n_mma;
            int tr[4] = {0, 0, 0, 0};
            if (gather_lane) {
#pragma unroll
                for (int j = 0; j < 4; ++j) tr[j] = token_row(p, ti.row0 + 4 * lane + j);
            }
            // token rows of this lane's scale factors: n = lane + 32 i
            int sf_tok[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int n = lane + 32 * i;
                sf_tok[i] = (n < BN && n < ti.n_mma) ? token_row(p, ti.row0 + n) : -1;
                if (sf_tok[i] >= mp.x_rows) sf_tok[i] = -1;
            }
            for (int kb = 0; kb < KB; ++kb) {
                if (lane == 0) ok = mbar_wait(&empty_bar[stage], phase ^ 1, abort_flag, p.err, 0);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                uint8_t *st = ring + stage * C::kStageBytes;
                uint8_t *sb = st + C::kABytes;
                uint8_t *sf = sb + C::kBBytes;
                // scale factors: weight rows m = lane + 32 i (gate, then up), then token rows
                for (int a = 0; a < C::kNumA; ++a) {
                    uint32_t v[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int row = a_row + (a ? p.m_out : 0) + lane + 32 * i;
                        v[i] = row < mp.w_total_rows
                                   ? __ldg(reinterpret_cast<const uint32_t *>(mp.w_sf + static_cast<size_t>(row) *
                                                                                         sf_row_bytes) + kb)
                                   : 0u;
                    }
                    *reinterpret_cast<uint4 *>(sf + a * kSfBlock + lane * 16) = make_uint4(v[0], v[1], v[2], v[3]);
                }
                {
                    uint32_t v[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        v[i] = sf_tok[i] >= 0
                                   ? __ldg(reinterpret_cast<const uint32_t *>(mp.x_sf + static_cast<size_t>(sf_tok[i]) *
                                                                                         sf_row_bytes) + kb)
                                   : 0u;
                    *reinterpret_cast<uint4 *>(sf + C::kNumA * kSfBlock + lane * 16) =
                        make_uint4(v[0], v[1], v[2], v[3]);
                }
                fence_proxy_async_smem();            // the tcgen05.cp of these bytes is an async-proxy read
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive_expect_tx(&full_bar[stage], tx);
                    tma_load_2d(st, &tmA, &full_bar[stage], kb * kMxBK, a_row, pol_w);
                    if (SWIGLU) tma_load_2d(st + kMxTileA, &tmA, &full_bar[stage], kb * kMxBK, a_row + p.m_out, pol_w);
                    if (!p.perm)
                        for (int b = 0; b < nbox; ++b)
                            tma_load_2d(sb + b * kBoxN * kMxBK, &tmB, &full_bar[stage], kb * kMxBK,
                                        ti.row0 + b * kBoxN, pol_x);
                }
                __syncwarp();
                if (gather_lane)
                    tma_gather4(sb + lane * 4 * kMxBK, &tmB, &full_bar[stage], kb * kMxBK, tr[0], tr[1], tr[2], tr[3],
                                pol_x);
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
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
            const uint32_t sf_col0 = tmem_base + 2 * C::kAccCols;
            for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
                const TileInfo ti = decode_tile(tile, pre_s, off_s, E, MB, BN);
                ok = mbar_wait(&tempty_bar[buf], bphase ^ 1, abort_flag, p.err);
                if (!ok) break;
                tc_fence_after_sync();
                const uint32_t d0 = tmem_base + buf * C::kAccCols;
                for (int kb = 0; kb < KB; ++kb) {
                    ok = mbar_wait(&full_bar[stage], phase, abort_flag, p.err, 0);
                    if (!ok) break;
                    tc_fence_after_sync();
                    const uint32_t st = smem_u32(ring + stage * C::kStageBytes);
                    const uint32_t sf = st + C::kABytes + C::kBBytes;
                    const uint32_t slot = sf_col0 + stage * C::kSfCols;   // this stage's TMEM scale columns
#pragma unroll
                    for (int a = 0; a <= C::kNumA; ++a)
                        tmem_cp_32x128b_warpx4(slot + 4 * a, sf_smem_desc(sf + a * kSfBlock));
                    const uint64_t db = sw128_kmajor_desc(st + C::kABytes);
#pragma unroll
                    for (int k = 0; k < kMxBK / 32; ++k) {
                        const uint32_t acc = (kb | k) != 0;
                        const uint32_t id = static_cast<uint32_t>(k);
                        const uint32_t idesc = idesc_mxf8f6f4(kBM, ti.n_mma, W4 ? kMxE2M1 : kMxE4M3, id, id);
                        const uint32_t sfb = (slot + 4 * C::kNumA) | (id << 30);
                        // +32 bytes per K step inside the swizzled row: +2 in the >>4 address field
                        umma_mxf8_ss(d0, sw128_kmajor_desc(st) + 2 * k, db + 2 * k, idesc, slot | (id << 30), sfb, acc);
                        if (SWIGLU)
                            umma_mxf8_ss(d0 + BN, sw128_kmajor_desc(st + kMxTileA) + 2 * k, db + 2 * k, idesc,
                                         (slot + 4) | (id << 30), sfb, acc);
                    }
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
    } else if (!SWIGLU) {
        // down: bf16 y rows, the weights-on-M epilogue
        run_epilogue<BN, false, C::kAccCols>(p, pre_s, off_s, total_tiles, MB, tmem_base, tfull_bar, tempty_bar,
                                             abort_flag, 128);
    } else {
        // gate/up: act = bf16(silu(g) * u), then MX-quantised along the
        // features: the 32 lanes of a warp hold 32 consecutive features of a
        // token, one MX block (I % 128 == 0, so every lane's feature exists)
        const int q = warp & 3;
        int buf = 0;
        uint32_t bphase = 0;
        const int I = p.m_out;
        for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
            const TileInfo ti = decode_tile(tile, pre_s, off_s, E, MB, BN);
            if (!mbar_wait(&tfull_bar[buf], bphase, abort_flag, p.err, 128)) break;
            tc_fence_after_sync();
            const int f = ti.mb * kBM + q * 32 + lane;
            const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * C::kAccCols;
            for (int c0 = 0; c0 < ti.n_mma; c0 += 16) {
                uint32_t g[16], u[16];
                tmem_ld_32x32b_x16(tb + c0, g);
                tmem_ld_32x32b_x16(tb + BN + c0, u);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int n = c0 + j;
                    if (n < ti.valid) {                      // warp-uniform
                        const float gv = __uint_as_float(g[j]);
                        const float a = gv / (1.0f + expf(-gv)) * __uint_as_float(u[j]);
                        const float ab = __bfloat162float(__float2bfloat16_rn(a));
                        const uint32_t amax = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(ab)));
                        const int e = mx_block_exponent(amax);
                        const size_t row = static_cast<size_t>(ti.row0 + n);
                        mp.out_q[row * I + f] = e4m3_rn_sat(__fmul_rn(ab, mx_inverse_scale(e)));
                        if (lane == 0) mp.out_sf[row * (I / 32) + (f >> 5)] = static_cast<uint8_t>(e + 127);
                    }
                }
            }
            tc_fence_before_sync();
            mbar_arrive(&tempty_bar[buf]);
            if (++buf == 2) { buf = 0; bphase ^= 1; }
        }
    }

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

template <int BN, int STAGES, bool SWIGLU, bool W4>
cudaError_t run_mx(const MxGemmArgs &g, cudaStream_t s) {
    using C = MxCfg<BN, STAGES, SWIGLU>;
    CUtensorMap ta, tb;
    const uint64_t a_rows = static_cast<uint64_t>(g.base.E) * g.base.w_rows;
    const uint64_t x_rows = g.base.perm ? static_cast<uint64_t>(g.base.T) : static_cast<uint64_t>(g.base.P);
    const uint64_t K = static_cast<uint64_t>(g.base.K);
    bool ok = (W4 ? make_map_pitched(&ta, g.base.w, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, K, a_rows, K / 2, kMxBK,
                                     kBM, CU_TENSOR_MAP_SWIZZLE_128B)
                  : make_map(&ta, g.base.w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, a_rows, kMxBK, kBM,
                             CU_TENSOR_MAP_SWIZZLE_128B)) &&
              make_map(&tb, g.base.a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, g.base.K, x_rows, kMxBK,
                       g.base.perm ? 1 : kBoxN, CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok) return cudaErrorInvalidValue;
    auto kern = grouped_gemm_mxfp8_kernel<BN, STAGES, SWIGLU, W4>;
    cudaError_t st = ensure_dynamic_smem(kern, C::kSmemBytes);
    if (st != cudaSuccess) return st;
    const int grid = grid_for(g.base, BN);
    if (grid <= 0) return cudaSuccess;
    MxParams mp;
    mp.p = make_params(g.base, BN);
    mp.w_sf = g.w_sf;
    mp.x_sf = g.x_sf;
    mp.out_q = g.out_q;
    mp.out_sf = g.out_sf;
    mp.w_total_rows = static_cast<int>(a_rows);
    mp.x_rows = static_cast<int>(x_rows);
    return launch_pdl(kern, dim3(grid), dim3(C::kThreads), C::kSmemBytes, s, ta, tb, mp);
}

template <bool W4>
cudaError_t dispatch_mx(const MxGemmArgs &g, cudaStream_t s) {
    const double avg = static_cast<double>(g.base.P) / g.base.E;
    if (g.base.swiglu) {
        if (avg <= 24) return run_mx<32, 4, true, W4>(g, s);
        return run_mx<64, 4, true, W4>(g, s);
    }
    if (avg <= 24) return run_mx<32, 6, false, W4>(g, s);
    if (avg <= 48) return run_mx<64, 6, false, W4>(g, s);
    return run_mx<128, 4, false, W4>(g, s);
}

}  // namespace

cudaError_t launch_grouped_gemm_mxfp8(const MxGemmArgs &g, cudaStream_t s) {
    if (g.base.P == 0) return cudaSuccess;
    if (g.base.fmt == 3) return dispatch_mx<true>(g, s);     // MXFP4 weights
    if (g.base.fmt != 2) return cudaErrorInvalidValue;
    return dispatch_mx<false>(g, s);
}

cudaError_t launch_mx_quantize(const uint16_t *x, int rows, int K, uint8_t *q, uint8_t *scales, cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    const long long total = static_cast<long long>(rows) * (K / 8);
    long long blocks = (total + 255) / 256;
    if (blocks > 148LL * 16) blocks = 148LL * 16;
    return launch_pdl(mx_quantize_kernel, dim3(static_cast<int>(blocks)), dim3(256), 0, s,
                      reinterpret_cast<const uint4 *>(x), total, reinterpret_cast<uint2 *>(q), scales);
}

}  // namespace moe
